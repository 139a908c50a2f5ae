// Fused selective-scan prefill for sm_100a.
//
// Page "SAMBA混合注意力状态空间模型", section 数学框架 / Mamba层: the Mamba
// layer's selective recurrence h_t = Ā_t h_{t-1} + B̄_t x_t, y_t = C_t h_t with
// input-dependent B_t, C_t and Δ_t = τ_Δ(·).  With the zero-order-hold decay
// Ā = exp(Δ A) (A diagonal, one value per channel and state), the Euler input
// term B̄x = Δ B u, the causal depthwise conv in front, the D skip and the
// silu(z) gate, each (batch, channel) runs
//
//   u_t   = SiLU(bias + sum_k w_k x_{t-K+1+k})
//   Δ_t   = softplus(delta_t)
//   h_t   = exp(Δ_t A) ⊙ h_{t-1} + Δ_t u_t B_t        (N states, fp32)
//   y_t   = (C_t · h_t + D u_t) · silu(z_t)
//
// The recurrence is sequential in t but independent across (batch, channel,
// state), and on B200 it is bound by arithmetic (one exp per state and token
// on a 16/clk/SM MUFU pipe), not by HBM.  So the kernel spends as few
// instructions as it can per (token, channel, state) and keeps every SM busy:
//
//   * A CTA owns CU consecutive channels of one batch row (CU chosen on the
//     host so that the CTAs spread evenly over the SMs) and walks the whole
//     sequence in tiles of T tokens.
//   * Warp roles.  One producer warp streams x, z, delta, B, C tiles into a
//     STAGES-deep shared-memory ring with TMA.  Prologue warps compute, once
//     per (token, channel), the conv, SiLU and softplus, leaving (Δ, Δu) for
//     the scan and (D·u, z) for the output.  The scan warps hold the state:
//     lane = channel, and each of the GL scan warps holds NS of a channel's N
//     states, so all lanes of a warp read the same B and C entries; each lane
//     writes its partial C·h per token.  Epilogue warps finish
//     y = (Σ partials + D·u)·silu(z) and store it.
//   * Prologue, scan and epilogue of consecutive tiles overlap through
//     SLOTS-deep exchange arrays guarded by mbarriers.
//   * The scan warps software-pipeline groups of G tokens: the decays
//     exp(Δ A) of group g+1, which do not depend on the state, are issued
//     next to the dependent updates of group g.  The core uses packed f32x2
//     arithmetic; a compile-time share of the exps can be evaluated on the
//     FMA pipe with a polynomial (exp2 split into 2^j · 2^f, degree-5 fit of
//     2^f on [-1/2, 1/2] with p(0) = 1 and p'(0) = ln 2).
//   * Every wait is bounded; a wait that runs out stops the CTA cleanly.
#include "common.cuh"

// Every SAMBA_SCAN_POLY-th token evaluates its exps on the FMA pipe
// (0: never).  A build-time constant, fixed by measurement.
#ifndef SAMBA_SCAN_POLY
#define SAMBA_SCAN_POLY 0
#endif
// States per scan lane at N = 16 (2 or 4); also fixed by measurement.
#ifndef SAMBA_SCAN_NS16
#define SAMBA_SCAN_NS16 4
#endif

namespace samba {

struct ScanParams {
  const float* A;
  const float* Dskip;
  const float* conv_w;
  const float* conv_b;
  const float* conv_state_in;
  float* conv_state_out;
  const float* h0;
  float* h_final;
  float* delta_sum;  // [B, D] sum over t of Δ, or null
  float* h_ckpt;     // [B, nck, N, D] state at the start of every 16-token chunk, or null
  int nck;           // ceil(L / 16)
  const void* x;  // for the conv state at the end
  void* y;
  int64_t L, D;
  int K;
  int CU;  // channels per CTA
  int has_z, fuse_conv, conv_silu, softplus;
};

template <int N> struct ScanShape;
template <> struct ScanShape<16> { static constexpr int NS = SAMBA_SCAN_NS16, GL = 16 / SAMBA_SCAN_NS16; };
template <> struct ScanShape<8> { static constexpr int NS = 1, GL = 8; };
template <> struct ScanShape<4> { static constexpr int NS = 1, GL = 4; };

constexpr int kScanCB = 32;     // channels in one TMA box (>= CU + alignment offset)
#ifndef SAMBA_SCAN_T
#define SAMBA_SCAN_T 32
#endif
constexpr int kScanT = SAMBA_SCAN_T;  // tokens per tile
// Prologue and epilogue warps (each a divisor of the tile's tokens).  Fixed by
// measurement: 4 prologue or 2 epilogue warps were slower, and so were 16
// prologue warps (fewer registers per thread).
#ifndef SAMBA_SCAN_PRO
#define SAMBA_SCAN_PRO 8
#endif
#ifndef SAMBA_SCAN_EPI
#define SAMBA_SCAN_EPI 8
#endif
constexpr int kScanPro = SAMBA_SCAN_PRO;  // prologue warps
// Upper bound on the block size (sets the register budget per thread).
#ifndef SAMBA_SCAN_MAXTHREADS
#define SAMBA_SCAN_MAXTHREADS 672
#endif
// Tokens per group of the scan warps' software pipeline.
#ifndef SAMBA_SCAN_GROUP
#define SAMBA_SCAN_GROUP 4
#endif
#ifndef SAMBA_SCAN_SLOTS
#define SAMBA_SCAN_SLOTS 4
#endif

constexpr int kScanSlots = SAMBA_SCAN_SLOTS;  // depth of the prologue -> scan -> epilogue hand-off
constexpr int kScanSmemBudget = 227 * 1024;
// Epilogue warps: SAMBA_SCAN_EPI, or 4 where that would take a block with gl
// scan warps past SAMBA_SCAN_MAXTHREADS (8 scan warps at N = 8).
__host__ __device__ constexpr int scan_epi_warps(int gl) {
  return (gl + kScanPro + SAMBA_SCAN_EPI + 1) * 32 <= SAMBA_SCAN_MAXTHREADS ? SAMBA_SCAN_EPI : 4;
}
static_assert((8 + kScanPro + 4 + 1) * 32 <= SAMBA_SCAN_MAXTHREADS, "scan block exceeds SAMBA_SCAN_MAXTHREADS");

template <int N, typename XT>
struct ScanLayout {
  static constexpr int GL = ScanShape<N>::GL;
  // tiles of kScanT tokens at N = 16; 32 at smaller N (more partials per channel)
  static constexpr int CB = kScanCB, T = N == 16 ? kScanT : 32, HALO = 3, SLOTS = kScanSlots;
  static constexpr int al(int v) { return (v + 127) / 128 * 128; }
  static constexpr int XB = (T + HALO) * CB * (int)sizeof(XT);
  static constexpr int ZB = T * CB * (int)sizeof(XT);
  static constexpr int WB = T * CB * 4;
  static constexpr int BB = T * N * 4;
  static constexpr int X_OFF = 0, Z_OFF = al(XB), W_OFF = Z_OFF + al(ZB), B_OFF = W_OFF + al(WB),
                       C_OFF = B_OFF + al(BB), STAGE_BYTES = C_OFF + al(BB);
  static constexpr int XCH_BYTES = SLOTS * T * CB * 8;       // float2 [SLOTS][T][CB] (Δ, Δu)
  static constexpr int EPI_BYTES = SLOTS * T * CB * 8;       // float2 [SLOTS][T][CB] (D·u, z)
  static constexpr int PART_BYTES = SLOTS * T * CB * GL * 4; // float  [SLOTS][T][GL][CB]
  // barriers (256 B), then the prologue's partial sums of Δ ([kScanPro][CB] floats)
  static constexpr int BAR_BYTES = 512 + kScanPro * CB * 4;
  static constexpr int FIXED = XCH_BYTES + EPI_BYTES + PART_BYTES + BAR_BYTES;
  // TMA ring: as many stages (up to 6) as fit next to the hand-off buffers
  static constexpr int STAGES_FIT = (kScanSmemBudget - FIXED) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 6 ? 6 : STAGES_FIT;
  static_assert(STAGES >= 2, "scan tile does not fit in shared memory");
  static constexpr int XCH_OFF = STAGES * STAGE_BYTES;
  static constexpr int EPI_OFF = XCH_OFF + XCH_BYTES;
  static constexpr int PART_OFF = EPI_OFF + EPI_BYTES;
  static constexpr int BAR_OFF = PART_OFF + PART_BYTES;
  static constexpr int SMEM = BAR_OFF + BAR_BYTES;
};

// Scan warps: one per group of NS states (GL of them); lane = channel (CU <= 32).
__host__ __device__ constexpr int scan_warps(int gl) { return gl; }

// ------------------------------------------------------------ math helpers
__device__ __forceinline__ float mufu_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float mufu_rcp(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA pipe for a pair of arguments: x = j + f with j = rint(x)
// (magic-number rounding), 2^f by a degree-5 polynomial fitted on
// [-1/2, 1/2] for relative error (fit made for this library; c0 = 1 and
// c1 = ln 2 are pinned so that 2^f - 1 stays accurate for tiny f), and the
// exponent j added to the bits of 2^f.  x is clamped to [-125, 127]; below
// that the true value is under 2^-125 and is returned as 2^-125.
__device__ __forceinline__ f2 ex2_poly2(f2 x) {
  float2 xv = up2(x);
  xv.x = fminf(fmaxf(xv.x, -125.f), 127.f);
  xv.y = fminf(fmaxf(xv.y, -125.f), 127.f);
  const f2 xc = pk2(xv.x, xv.y);
  const f2 magic = pk2(12582912.f, 12582912.f);  // 1.5 * 2^23
  const f2 t = add2(xc, magic);
  const f2 j = sub2(t, magic);
  const f2 f = sub2(xc, j);
  f2 p = pk2(0x1.59c4aap-10f, 0x1.59c4aap-10f);
  p = fma2(p, f, pk2(0x1.3c6c98p-7f, 0x1.3c6c98p-7f));
  p = fma2(p, f, pk2(0x1.c6b7f4p-5f, 0x1.c6b7f4p-5f));
  p = fma2(p, f, pk2(0x1.ebfb30p-3f, 0x1.ebfb30p-3f));
  p = fma2(p, f, pk2(0x1.62e430p-1f, 0x1.62e430p-1f));
  p = fma2(p, f, pk2(1.f, 1.f));
  const float2 tv = up2(t), pv = up2(p);
  const float r0 = __int_as_float(__float_as_int(pv.x) + (__float_as_int(tv.x) << 23));
  const float r1 = __int_as_float(__float_as_int(pv.y) + (__float_as_int(tv.y) << 23));
  return pk2(r0, r1);
}

__device__ __forceinline__ float silu_fast(float v) {
  return v * mufu_rcp(1.0f + mufu_ex2(v * -1.4426950408889634f));
}

// softplus(w) = log(1 + e^w).  For w <= 0 with e = e^w: log1p(e) = 2 atanh(s),
// s = e / (2 + e) in (0, 1/3], summed as 2s(1 + s²/3 + ... + s¹²/13) (the
// next term is below 1.5e-8 relative).  For w > 0 the identity
// softplus(w) = w + softplus(-w) is used, and for w > 20 softplus(w) = w in
// fp32.
__device__ __forceinline__ float softplus_fast(float w) {
  const float e = mufu_ex2(-fabsf(w) * 1.4426950408889634f);
  const float s = e * mufu_rcp(2.0f + e);
  const float s2 = s * s;
  float p = 1.f / 13.f;
  p = fmaf(p, s2, 1.f / 11.f);
  p = fmaf(p, s2, 1.f / 9.f);
  p = fmaf(p, s2, 1.f / 7.f);
  p = fmaf(p, s2, 1.f / 5.f);
  p = fmaf(p, s2, 1.f / 3.f);
  p = fmaf(p, s2, 1.f);
  const float l = 2.f * s * p;
  return w > 20.f ? w : (w > 0.f ? w + l : l);
}

// ------------------------------------------------------------------ kernel
// Warp roles (index ranges): [0, NSW) scan, then kScanPro prologue, then
// EPIW epilogue, then one TMA producer.  Per tile i (slot k = i % SLOTS):
//   producer : full[s] <- TMA of x, z, delta, B, C          (waits empty[s])
//   prologue : XCH[k], EPI[k] <- conv/softplus, D·u, z; arrives pro_full[k]
//              (waits full[s]; scan_done[k] and epi_done[k] of tile i-SLOTS)
//   scan     : PART[k] <- partial C·h of its states; arrives scan_done[k]
//              (waits pro_full[k], full[s]; pro_full[k] follows the
//              prologue's own wait for epi_done[k] of tile i-SLOTS)
//   epilogue : y <- (Σ PART[k] + D·u)·silu(z); arrives epi_done[k]
//              (waits scan_done[k])
// empty[s] collects the prologue and scan warps (the readers of stage s).
template <int N, typename XT, typename YT, int POLY, bool CKPT>
__global__ void __launch_bounds__(SAMBA_SCAN_MAXTHREADS, 1)
    scan_fwd_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_z,
                    const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_b,
                    const __grid_constant__ CUtensorMap map_c, const ScanParams p) {
  using Ly = ScanLayout<N, XT>;
  constexpr int NS = ScanShape<N>::NS, GL = ScanShape<N>::GL;
  constexpr int T = Ly::T, CB = Ly::CB, STAGES = Ly::STAGES, HALO = Ly::HALO, SLOTS = Ly::SLOTS;
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Ly::BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* pro_full = empty + STAGES;      // [SLOTS]
  uint64_t* scan_done = pro_full + SLOTS;   // [SLOTS]
  uint64_t* epi_done = scan_done + SLOTS;   // [SLOTS]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(epi_done + SLOTS);
  uint64_t* dsum_bar = reinterpret_cast<uint64_t*>(smem + Ly::BAR_OFF + 256);  // partial Δ sums written
  float* DSUM = reinterpret_cast<float*>(smem + Ly::BAR_OFF + 512);            // [kScanPro][CB]
  float2* XCH = reinterpret_cast<float2*>(smem + Ly::XCH_OFF);
  float2* EPI = reinterpret_cast<float2*>(smem + Ly::EPI_OFF);
  float* PART = reinterpret_cast<float*>(smem + Ly::PART_OFF);

  const int CU = p.CU;
  constexpr int NSW = scan_warps(GL), EPIW = scan_epi_warps(GL);
  const int PRO0 = NSW, EPI0 = NSW + kScanPro, PROD = NSW + kScanPro + EPIW;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int c_start = blockIdx.x * CU;
  const int c_box = c_start & ~7;
  const int off = c_start - c_box;
  const int64_t L = p.L;
  const int ntiles = static_cast<int>((L + T - 1) / T);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NSW + kScanPro);
    }
    for (int k = 0; k < SLOTS; ++k) {
      mbar_init(&pro_full[k], kScanPro);
      mbar_init(&scan_done[k], NSW);
      mbar_init(&epi_done[k], EPIW);
    }
    mbar_init(dsum_bar, kScanPro - 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == PROD) {
    // ================================================================ TMA
    if (lane == 0) {
      tma_prefetch_desc(&map_x);
      tma_prefetch_desc(&map_w);
      tma_prefetch_desc(&map_b);
      tma_prefetch_desc(&map_c);
      if (p.has_z) tma_prefetch_desc(&map_z);
      const uint32_t bytes = Ly::XB + (p.has_z ? Ly::ZB : 0) + Ly::WB + 2 * Ly::BB;
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % STAGES;
        if (i >= STAGES && !mbar_wait(&empty[s], ((i / STAGES) - 1) & 1, abort_flag)) break;
        unsigned char* st = smem + s * Ly::STAGE_BYTES;
        const int t0 = i * T;
        mbar_arrive_expect_tx(&full[s], bytes);
        tma_load_3d(st + Ly::X_OFF, &map_x, &full[s], c_box, t0 - HALO, b);
        if (p.has_z) tma_load_3d(st + Ly::Z_OFF, &map_z, &full[s], c_box, t0, b);
        tma_load_3d(st + Ly::W_OFF, &map_w, &full[s], c_box, t0, b);
        tma_load_3d(st + Ly::B_OFF, &map_b, &full[s], 0, t0, b);
        tma_load_3d(st + Ly::C_OFF, &map_c, &full[s], 0, t0, b);
        issued = i + 1;
      }
      for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i) {
        volatile int never = 0;
        mbar_wait(&full[i % STAGES], (i / STAGES) & 1, &never);
      }
    }
    return;
  }

  if (warp >= EPI0) {
    // ============================================================ epilogue
    // Thread (eg, cl): channel cl (lane), tokens [eg·TPE, (eg+1)·TPE) of every tile.
    constexpr int TPE = T / EPIW;
    const int cl = lane, eg = warp - EPI0;
    const int64_t c = c_start + cl;
    const bool cval = cl < CU && c < p.D;
    for (int i = 0; i < ntiles; ++i) {
      const int k = i % SLOTS, r = i / SLOTS;
      const bool ok = mbar_wait(&scan_done[k], r & 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      const int64_t t0 = (int64_t)i * T;
      float4 pv[TPE];
      float2 ev[TPE];
#pragma unroll
      for (int q = 0; q < TPE; ++q) {
        const int t = eg * TPE + q;
        const float* part = PART + (k * T + t) * GL * CB + cl;
        pv[q] = make_float4(part[0], part[CB], part[2 * CB], part[3 * CB]);
        if (GL == 8) {
          pv[q].x += part[4 * CB];
          pv[q].y += part[5 * CB];
          pv[q].z += part[6 * CB];
          pv[q].w += part[7 * CB];
        }
        ev[q] = EPI[(k * T + t) * CB + cl];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&epi_done[k]);
#pragma unroll
      for (int q = 0; q < TPE; ++q) {
        const int64_t tok = t0 + eg * TPE + q;
        const float acc = (pv[q].x + pv[q].y) + (pv[q].z + pv[q].w);
        const float g = p.has_z ? silu_fast(ev[q].y) : 1.f;
        const int64_t yi = ((int64_t)b * L + tok) * p.D + c;
        if (cval && tok < L && SAMBA_CHECK(yi >= 0 && yi < (int64_t)gridDim.y * L * p.D))
          reinterpret_cast<YT*>(p.y)[yi] = from_f32<YT>((acc + ev[q].x) * g);
      }
    }
    return;
  }

  if (warp >= PRO0) {
    // ============================================================ prologue
    // Thread (tg, cl): channel cl of the CTA (lane), tokens [tg·TPT, (tg+1)·TPT)
    // of every tile, so its per-channel constants stay in registers and the
    // conv taps slide along consecutive tokens.
    constexpr int TPT = T / kScanPro;  // tokens per thread per tile
    const int cl = lane;
    const int tg = warp - PRO0;
    const int cb = off + cl;
    const int64_t c = c_start + cl;
    const bool cact = cl < CU;           // lane owns a channel of this CTA
    const bool cval = cact && c < p.D;   // ... that exists
    const int K = p.K;
    float cw[4] = {0.f, 0.f, 0.f, 0.f};
    float cbias = 0.f, dsk = 0.f;
    float hist[3] = {0.f, 0.f, 0.f};  // x of the 3 tokens before the first tile (conv state)
    float dsum = 0.f;                 // sum of Δ over this thread's tokens (0 for padding tokens)
    if (cval) {
      if (p.fuse_conv) {
        // tap k (0..3) multiplies x_{t-3+k}: weight k - (4 - K), if any
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int kk = k - (4 - K);
          cw[k] = kk >= 0 ? p.conv_w[c * K + kk] : 0.f;
        }
        if (p.conv_b) cbias = p.conv_b[c];
        if (p.conv_state_in) {
#pragma unroll
          for (int k = 0; k < 3; ++k) {  // hist[k] = x_{k-3}: state entry k - (4 - K)
            const int kk = k - (4 - K);
            hist[k] = kk >= 0 ? p.conv_state_in[((int64_t)b * p.D + c) * (K - 1) + kk] : 0.f;
          }
        }
      }
      if (p.Dskip) dsk = p.Dskip[c];
    }

    for (int i = 0; i < ntiles; ++i) {
      const int s = i % STAGES, k = i % SLOTS, r = i / SLOTS;
      bool ok = mbar_wait(&full[s], (i / STAGES) & 1, abort_flag);
      if (r >= 1) {
        ok = ok && mbar_wait(&scan_done[k], (r - 1) & 1, abort_flag);
        ok = ok && mbar_wait(&epi_done[k], (r - 1) & 1, abort_flag);
      }
      if (!__all_sync(0xffffffffu, ok)) break;
      const unsigned char* st = smem + s * Ly::STAGE_BYTES;
      const XT* xs = reinterpret_cast<const XT*>(st + Ly::X_OFF);
      const XT* zs = reinterpret_cast<const XT*>(st + Ly::Z_OFF);
      const float* ws = reinterpret_cast<const float*>(st + Ly::W_OFF);
      const int64_t t0 = (int64_t)i * T;
      const int tb = tg * TPT;  // first token of this thread in the tile
      // conv window: smem row r holds token t0 - 3 + r
      float xw[TPT + 3], wv[TPT], zv[TPT];
#pragma unroll
      for (int q = 0; q < TPT + 3; ++q) xw[q] = to_f32<XT>(xs[(tb + q) * CB + cb]);
#pragma unroll
      for (int q = 0; q < TPT; ++q) {
        wv[q] = ws[(tb + q) * CB + cb];
        zv[q] = p.has_z ? to_f32<XT>(zs[(tb + q) * CB + cb]) : 0.f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);  // x, z, delta of stage s consumed
      if (i == 0 && tb == 0) {  // tokens before the sequence come from the conv state
        xw[0] = hist[0];
        xw[1] = hist[1];
        xw[2] = hist[2];
      }
#pragma unroll
      for (int q = 0; q < TPT; ++q) {
        const int t = tb + q;
        const int64_t tok = t0 + t;
        float u;
        if (p.fuse_conv) {
          float acc = cbias;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) acc = fmaf(cw[kk], xw[q + kk], acc);
          u = p.conv_silu ? silu_fast(acc) : acc;
        } else {
          u = xw[q + HALO];
        }
        const float wr = wv[q];
        float dlt = p.softplus ? softplus_fast(wr) : wr;
        if (tok >= L || !cact) dlt = 0.f;  // padding tokens leave the state untouched
        const float du = dlt * u;
        dsum += dlt;
        // z itself goes to the epilogue warps, which wait on the scan most
        // of the time and evaluate the gate silu(z) there
        const float g = p.has_z ? zv[q] : 1.f;
        if (cact) {
          XCH[(k * T + t) * CB + cl] = make_float2(dlt, du);
          EPI[(k * T + t) * CB + cl] = make_float2(dsk * u, g);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&pro_full[k]);
    }
    if (*abort_flag) return;
    // Σ_t Δ per channel: each prologue warp holds the sums of its tokens; the
    // first one adds them in warp order once the others have written theirs.
    if (p.delta_sum) {
      DSUM[tg * CB + cl] = dsum;
      if (tg != 0) {
        __syncwarp();
        if (lane == 0) mbar_arrive(dsum_bar);
      } else {
        const bool ok = __all_sync(0xffffffffu, mbar_wait(dsum_bar, 0, abort_flag));
        if (ok && cval) {
          float sum = 0.f;
#pragma unroll
          for (int w = 0; w < kScanPro; ++w) sum += DSUM[w * CB + cl];
          p.delta_sum[(int64_t)b * p.D + c] = sum;
        }
      }
    }
    // final conv state: the last K-1 entries of (old state, x)
    if (p.conv_state_out && cval && tg == 0) {
      for (int jj = 0; jj < K - 1; ++jj) {
        const int64_t src = L + jj - (K - 1);
        float v;
        if (src >= 0) v = to_f32<XT>(reinterpret_cast<const XT*>(p.x)[((int64_t)b * L + src) * p.D + c]);
        else v = p.conv_state_in ? p.conv_state_in[((int64_t)b * p.D + c) * (K - 1) + (K - 1) + src] : 0.f;
        p.conv_state_out[((int64_t)b * p.D + c) * (K - 1) + jj] = v;
      }
    }
    return;
  }

  // ==================================================================== scan
  // Warp j, lane cl: channel cl of the CTA, states [j·NS, (j+1)·NS) held as
  // NP packed pairs.  Every lane of a warp reads the same B and C entries of
  // a token (a shared-memory broadcast).  Lanes past the CTA's channels run
  // along on zeros and write no partials.
  constexpr int NP = (NS + 1) / 2;
  const int j = warp, cl = lane;
  const int64_t c = c_start + cl;
  const bool cown = cl < CU;  // lane owns a channel
  const bool cval = cown && c < p.D;
  const int n0 = j * NS;
  constexpr float kLog2e = 1.4426950408889634f;
  f2 a2p[NP], hp[NP];
#pragma unroll
  for (int q = 0; q < NP; ++q) {
    float a[2] = {0.f, 0.f}, hh[2] = {0.f, 0.f};
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int n = n0 + 2 * q + r;
      if (2 * q + r < NS && cval) {
        a[r] = p.A[c * N + n] * kLog2e;
        if (p.h0) hh[r] = p.h0[((int64_t)b * p.D + c) * N + n];
      }
    }
    a2p[q] = pk2(a[0], a[1]);
    hp[q] = pk2(hh[0], hh[1]);
  }
  // checkpoint cidx: the state before token 16 * cidx ([b][cidx][n][D])
  auto store_ckpt = [&](int64_t cidx) {
    if (!cval || cidx >= p.nck) return;
    if (!SAMBA_CHECK(b < (int64_t)gridDim.y && c < p.D && n0 + NS <= N)) return;
    float* dst = p.h_ckpt + ((int64_t)b * p.nck + cidx) * N * p.D + c;
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      const float2 hv = up2(hp[q]);
      dst[(int64_t)(n0 + 2 * q) * p.D] = hv.x;
      if (2 * q + 1 < NS) dst[(int64_t)(n0 + 2 * q + 1) * p.D] = hv.y;
    }
  };
  static_assert(T % 16 == 0, "tiles hold whole 16-token chunks");
  if constexpr (CKPT) store_ckpt(0);

  for (int i = 0; i < ntiles; ++i) {
    const int s = i % STAGES, k = i % SLOTS, r = i / SLOTS;
    // PART[k] may be rewritten once the epilogue has read tile i - SLOTS:
    // the prologue waits for that (epi_done[k]) before it arrives on
    // pro_full[k], so the wait on pro_full[k] covers it.
    bool ok = mbar_wait(&pro_full[k], r & 1, abort_flag);
    ok = ok && mbar_wait(&full[s], (i / STAGES) & 1, abort_flag);
    if (!__all_sync(0xffffffffu, ok)) break;
    const unsigned char* st = smem + s * Ly::STAGE_BYTES;
    const float* bs = reinterpret_cast<const float*>(st + Ly::B_OFF);
    const float* cs = reinterpret_cast<const float*>(st + Ly::C_OFF);
    const float2* xch = XCH + k * T * CB + cl;
    float* part = PART + (k * T * GL + j) * CB + cl;
    constexpr int G = SAMBA_SCAN_GROUP;
    // B and C of token t for this lane's states, as packed pairs.
    auto load_bc = [&](int t, f2 (&bq)[NP], f2 (&cq)[NP]) {
      if (NS == 4) {
        const float4 bv = *reinterpret_cast<const float4*>(bs + t * N + n0);
        const float4 cv = *reinterpret_cast<const float4*>(cs + t * N + n0);
        bq[0] = pk2(bv.x, bv.y);
        bq[NP - 1] = pk2(bv.z, bv.w);
        cq[0] = pk2(cv.x, cv.y);
        cq[NP - 1] = pk2(cv.z, cv.w);
      } else if (NS == 2) {
        const float2 bv = *reinterpret_cast<const float2*>(bs + t * N + n0);
        const float2 cv = *reinterpret_cast<const float2*>(cs + t * N + n0);
        bq[0] = pk2(bv.x, bv.y);
        cq[0] = pk2(cv.x, cv.y);
      } else {
        bq[0] = pk2(bs[t * N + n0], 0.f);
        cq[0] = pk2(cs[t * N + n0], 0.f);
      }
    };
    // exp(Δ A) for this lane's states (A pre-scaled by log2 e).
    auto decay = [&](float dlt, int q, f2 (&dq)[NP]) {
      const f2 dlt2 = pk2(dlt, dlt);
#pragma unroll
      for (int m = 0; m < NP; ++m) {
        const f2 xx = mul2(dlt2, a2p[m]);
        if (POLY > 0 && (q % (POLY > 0 ? POLY : 1)) == POLY - 1) {
          dq[m] = ex2_poly2(xx);
        } else {
          const float2 xv = up2(xx);
          dq[m] = pk2(mufu_ex2(xv.x), NS >= 2 ? mufu_ex2(xv.y) : 0.f);
        }
      }
    };
    // h <- exp(Δ A) h + Δu B for one token; returns this lane's part of C·h.
    auto update = [&](const f2 (&dq)[NP], float du, const f2 (&bq)[NP], const f2 (&cq)[NP]) {
      const f2 du2 = pk2(du, du);
      f2 acc;
#pragma unroll
      for (int m = 0; m < NP; ++m) {
        hp[m] = fma2(dq[m], hp[m], mul2(du2, bq[m]));
        acc = m == 0 ? mul2(cq[m], hp[m]) : fma2(cq[m], hp[m], acc);
      }
      const float2 pr = up2(acc);
      return pr.x + pr.y;
    };
    {
      // Software pipeline over groups of G tokens: the decays of group g+1
      // (MUFU, independent of the state) are issued next to the dependent
      // updates of group g, so the special-function pipe is fed steadily.
      constexpr int NG = T / G;
      float2 evn[G];
      f2 dAn[G][NP];
#pragma unroll
      for (int q = 0; q < G; ++q) evn[q] = xch[q * CB];
#pragma unroll
      for (int q = 0; q < G; ++q) decay(evn[q].x, q, dAn[q]);
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        const int tg0 = g * G;
        float duc[G];
        f2 dAc[G][NP];
#pragma unroll
        for (int q = 0; q < G; ++q) {
          duc[q] = evn[q].y;
#pragma unroll
          for (int m = 0; m < NP; ++m) dAc[q][m] = dAn[q][m];
        }
        if (g + 1 < NG) {
#pragma unroll
          for (int q = 0; q < G; ++q) evn[q] = xch[(tg0 + G + q) * CB];
        }
        f2 bb[G][NP], cc[G][NP];
#pragma unroll
        for (int q = 0; q < G; ++q) load_bc(tg0 + q, bb[q], cc[q]);
        if (g + 1 < NG) {
#pragma unroll
          for (int q = 0; q < G; ++q) decay(evn[q].x, q, dAn[q]);
        }
        float pv[G];
#pragma unroll
        for (int q = 0; q < G; ++q) pv[q] = update(dAc[q], duc[q], bb[q], cc[q]);
#pragma unroll
        for (int q = 0; q < G; ++q)
          if (cown) part[(tg0 + q) * CB * GL] = pv[q];  // idle lanes would alias other channels
        if constexpr (CKPT) {
          if ((tg0 + G) % 16 == 0) store_ckpt(((int64_t)i * T + tg0 + G) / 16);
        }
      }
    }
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&scan_done[k]);
      mbar_arrive(&empty[s]);
    }
  }
  if (*abort_flag) return;
  if (cval && p.h_final && SAMBA_CHECK(b < (int64_t)gridDim.y && c < p.D && n0 + NS <= N)) {
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      const float2 hv = up2(hp[q]);
      p.h_final[((int64_t)b * p.D + c) * N + n0 + 2 * q] = hv.x;
      if (2 * q + 1 < NS) p.h_final[((int64_t)b * p.D + c) * N + n0 + 2 * q + 1] = hv.y;
    }
  }
}

}  // namespace samba

// ------------------------------------------------------------------- launcher
#include "host.hpp"

namespace samba {

int take_status_scan(cudaStream_t s) { return take_status_word(s); }

// Channels per CTA: the largest multiple of 4 (<= 32, and <= 28 unless a
// multiple of 8 so that the 16-byte-aligned TMA box of 32 channels covers it)
// that minimises (waves of CTAs) x (channels per CTA) on this GPU.
static int choose_cu(int64_t B, int64_t D) {
  const int sms = sm_count();
  int best = 32;
  int64_t best_cost = INT64_MAX;
  for (int cu = 32; cu >= 8; cu -= 4) {
    if (cu % 8 != 0 && cu > 28) continue;
    const int64_t ctas = B * ((D + cu - 1) / cu);
    const int64_t waves = (ctas + sms - 1) / sms;
    const int64_t cost = waves * cu;
    if (cost < best_cost) {
      best_cost = cost;
      best = cu;
    }
  }
  return best;
}

// CKPT: the variant that also stores the chunk checkpoints (a separate
// instantiation, so that the kernel without them is unchanged).
template <int N, typename XT, typename YT, bool CKPT>
static int launch_scan_t(const samba_scan_args& a, cudaStream_t stream) {
  using Ly = ScanLayout<N, XT>;
  constexpr int POLY = SAMBA_SCAN_POLY;
  auto kern = scan_fwd_kernel<N, XT, YT, POLY, CKPT>;
  static PerDeviceOnce attr;
  const int arc = once_per_device(attr, [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::SMEM) == cudaSuccess
               ? SAMBA_OK
               : fail(SAMBA_ERR_CUDA, "scan: cannot set shared memory size");
  });
  if (arc != SAMBA_OK) return arc;
  const int CU = choose_cu(a.batch, a.dim);
  const uint64_t Bsz = a.batch, L = a.seqlen, D = a.dim;
  const uint32_t xs = sizeof(XT);
  const CUtensorMapDataType xdt = sizeof(XT) == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap mx, mz, mw, mb, mc;
  {
    const uint64_t dims[3] = {D, L, Bsz};
    const uint64_t st[2] = {D * xs, L * D * xs};
    const uint32_t boxx[3] = {(uint32_t)Ly::CB, (uint32_t)(Ly::T + Ly::HALO), 1};
    const uint32_t boxz[3] = {(uint32_t)Ly::CB, (uint32_t)Ly::T, 1};
    int rc = encode_tiled(&mx, xdt, 3, a.x, dims, st, boxx, CU_TENSOR_MAP_SWIZZLE_NONE, "scan x");
    if (rc) return rc;
    rc = encode_tiled(&mz, xdt, 3, a.z ? a.z : a.x, dims, st, boxz, CU_TENSOR_MAP_SWIZZLE_NONE, "scan z");
    if (rc) return rc;
    const uint64_t stw[2] = {D * 4, L * D * 4};
    rc = encode_tiled(&mw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, a.delta, dims, stw, boxz, CU_TENSOR_MAP_SWIZZLE_NONE,
                      "scan delta");
    if (rc) return rc;
    const uint64_t dimb[3] = {(uint64_t)N, L, Bsz};
    const uint64_t stb[2] = {(uint64_t)N * 4, L * N * 4};
    const uint32_t boxb[3] = {(uint32_t)N, (uint32_t)Ly::T, 1};
    rc = encode_tiled(&mb, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, a.Bm, dimb, stb, boxb, CU_TENSOR_MAP_SWIZZLE_NONE, "scan B");
    if (rc) return rc;
    rc = encode_tiled(&mc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, a.Cm, dimb, stb, boxb, CU_TENSOR_MAP_SWIZZLE_NONE, "scan C");
    if (rc) return rc;
  }
  ScanParams p;
  p.A = a.A;
  p.Dskip = a.Dskip;
  p.conv_w = a.conv_w;
  p.conv_b = a.conv_b;
  p.conv_state_in = a.conv_state_in;
  p.conv_state_out = a.conv_state_out;
  p.h0 = a.h0;
  p.h_final = a.h_final;
  p.delta_sum = a.delta_sum;
  p.h_ckpt = a.h_ckpt;
  p.nck = static_cast<int>((a.seqlen + 15) / 16);
  p.x = a.x;
  p.y = a.y;
  p.L = a.seqlen;
  p.D = a.dim;
  p.K = a.dconv;
  p.CU = CU;
  p.has_z = a.z != nullptr;
  p.fuse_conv = (a.flags & SAMBA_SCAN_FUSE_CONV) != 0;
  p.conv_silu = (a.flags & SAMBA_SCAN_CONV_SILU) != 0;
  p.softplus = (a.flags & SAMBA_SCAN_DELTA_SOFTPLUS) != 0;
  constexpr int GLN = ScanShape<N>::GL;
  const int threads = (scan_warps(GLN) + kScanPro + scan_epi_warps(GLN) + 1) * 32;
  static_assert((scan_warps(GLN) + kScanPro + scan_epi_warps(GLN) + 1) * 32 <= SAMBA_SCAN_MAXTHREADS,
                "scan block exceeds SAMBA_SCAN_MAXTHREADS");
  dim3 grid((unsigned)((D + CU - 1) / CU), (unsigned)Bsz);
  kern<<<grid, threads, Ly::SMEM, stream>>>(mx, mz, mw, mb, mc, p);
  return check_launch("samba_selective_scan_fwd");
}

template <int N, bool CKPT>
static int launch_scan_c(const samba_scan_args& a, cudaStream_t s) {
  const bool xb = a.x_dtype == SAMBA_BF16, yb = a.y_dtype == SAMBA_BF16;
  if (xb && yb) return launch_scan_t<N, __nv_bfloat16, __nv_bfloat16, CKPT>(a, s);
  if (xb && !yb) return launch_scan_t<N, __nv_bfloat16, float, CKPT>(a, s);
  if (!xb && yb) return launch_scan_t<N, float, __nv_bfloat16, CKPT>(a, s);
  return launch_scan_t<N, float, float, CKPT>(a, s);
}

template <int N>
static int launch_scan_n(const samba_scan_args& a, cudaStream_t s) {
  return a.h_ckpt ? launch_scan_c<N, true>(a, s) : launch_scan_c<N, false>(a, s);
}

int launch_scan(const samba_scan_args& a, cudaStream_t s) {
  if (a.z && a.z_dtype != a.x_dtype)
    return fail(SAMBA_ERR_UNSUPPORTED, "samba_selective_scan_fwd: z dtype must equal x dtype");
  switch (a.dstate) {
    case 4: return launch_scan_n<4>(a, s);
    case 8: return launch_scan_n<8>(a, s);
    default: return launch_scan_n<16>(a, s);
  }
}

}  // namespace samba
