// Backward of banded sliding-window attention on the sm_100a tensor cores:
// dq, dk, dv from dO, given q, k, v, the forward's output o and its
// log-sum-exp.
//
// Page "SAMBA混合注意力状态空间模型", section 滑动窗口注意力: o = softmax(Q Kᵀ
// · scale + M) V with the window mask read as the causal band 0 <= i - j < W
// (grouped kv heads).  With P the softmax and dO = ∂L/∂o, per query row i and
// head h:  dV_j += P_ij dO_i,  dP_ij = dO_i · v_j,  dS_ij = P_ij (dP_ij - D_i)
// with D_i = Σ_j P_ij dP_ij = dO_i · o_i,  dq_i = scale Σ_j dS_ij k_j,
// dk_j += scale dS_ij q_i; a kv head's gradients sum over its query heads.
// P is recomputed from the scores and the stored log-sum-exp.
//
// Three kernels:
//   * swa_bwd_prep: per (b, token, head) the log-sum-exp in base 2 and D,
//     written in the order the 128-row tiles read them (the GROUP heads of a
//     kv head stacked per token, as the forward stacks its Q tiles), padded
//     with (+inf, 0) past the sequence so padded rows get P = 0;
//   * swa_bwd_kv_kernel: one CTA per (b, kv head, 128-key tile).  K and V stay
//     in shared memory; the Q/dO tiles of the band (TOK tokens x GROUP heads
//     each) stream through a TMA ring.  Per tile the MMA warp computes
//     Sᵀ = K Qᵀ and dPᵀ = V dOᵀ into tensor memory, the four compute warps
//     (thread = key) turn them into Pᵀ and dSᵀ (bf16, back into tensor
//     memory), and the MMA warp accumulates dV += Pᵀ dO and dK += dSᵀ Q with
//     A read from tensor memory;
//   * swa_bwd_q_kernel: one CTA per (b, kv head, TOK tokens): S = Q Kᵀ,
//     dP = dO Vᵀ over the key tiles of the band, dS on the compute warps
//     (thread = query row), dQ += dS K.
// Every MMA is kind::f16 (bf16 operands, fp32 accumulation) in the forms the
// forward kernel uses: both operands K-major from shared memory, or A from
// tensor memory and B MN-major from shared memory.  Every wait is bounded.
#include <cmath>

#include "common.cuh"
#include "host.hpp"

namespace samba {

int take_status_swa_bwd(cudaStream_t s) { return take_status_word(s); }

namespace {

constexpr float kLog2eB = 1.4426950408889634f;

__device__ __forceinline__ float ex2b(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

struct SwaBwdParams {
  const __nv_bfloat16* o;
  const __nv_bfloat16* dO;
  const float* lse;        // [B, Hq, L] natural log (forward output)
  float* lse2s;            // [B, Hkv, Lp, GROUP]  lse · log2(e)
  float* Ds;               // [B, Hkv, Lp, GROUP]  dO · o
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int64_t L, Lp, W;
  int Hq, Hkv, B;
  float scale, scale_log2;
  int ktiles;              // 128-key tiles per (b, kv head)
  int qtiles;              // TOK-token query tiles per (b, kv head)
};

// ------------------------------------------------------------------ prep
template <int HD>
__global__ void __launch_bounds__(256) swa_bwd_prep_kernel(const SwaBwdParams p, int group) {
  const int64_t n = static_cast<int64_t>(p.B) * p.Lp * p.Hq;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int h = static_cast<int>(e % p.Hq);
    const int64_t i = (e / p.Hq) % p.Lp;
    const int64_t b = e / (static_cast<int64_t>(p.Hq) * p.Lp);
    float lse2 = INFINITY, dsum = 0.f;
    if (i < p.L) {
      const int64_t row = ((b * p.L + i) * p.Hq + h) * HD;
      const uint4* a = reinterpret_cast<const uint4*>(p.o + row);
      const uint4* c = reinterpret_cast<const uint4*>(p.dO + row);
#pragma unroll
      for (int v = 0; v < HD / 8; ++v) {
        const uint4 x = a[v], y = c[v];
        const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          dsum = fmaf(__uint_as_float(xs[k] << 16), __uint_as_float(ys[k] << 16), dsum);
          dsum = fmaf(__uint_as_float(xs[k] & 0xFFFF0000u), __uint_as_float(ys[k] & 0xFFFF0000u), dsum);
        }
      }
      lse2 = p.lse[(b * p.Hq + h) * p.L + i] * kLog2eB;
    }
    const int g = h / group, hh = h % group;
    const int64_t dst = ((b * p.Hkv + g) * p.Lp + i) * group + hh;
    p.lse2s[dst] = lse2;
    p.Ds[dst] = dsum;
  }
}

// --------------------------------------------------------------- configs
template <int HD, int GROUP>
struct BwdCfg {
  static constexpr int TOK = 128 / GROUP;
  static constexpr int ROW_BYTES = HD * 2;
  static constexpr int TILE_BYTES = 128 * ROW_BYTES;
  static constexpr uint32_t SWZ = HD == 64 ? 2u : (HD == 32 ? 4u : 6u);
  static constexpr uint32_t ATOM = 8 * ROW_BYTES;
  // NCW compute warps per tensor-memory lane quarter (warp w reads lanes
  // 32 (w % 4) ..), each taking 128 / NCW of the tile's columns, so that
  // every sub-partition runs NCW independent exp chains.
  static constexpr int NCW = 4;
  static constexpr int CWARPS = 4 * NCW;
  static constexpr int CW = 128 / NCW;             // columns per compute warp
  static_assert(CW == 32, "one 32-column chunk per compute warp");
  static constexpr int WARP_TMA = CWARPS, WARP_MMA = CWARPS + 1;
  static constexpr int THREADS = 32 * (CWARPS + 2);
};

// dK/dV kernel shared memory: K, V; STG stages of (Q, dO, lse2[128], D[128]).
template <int HD, int GROUP, int STG>
struct KvCfg : BwdCfg<HD, GROUP> {
  using B_ = BwdCfg<HD, GROUP>;
  static constexpr int K_OFF = 0, V_OFF = B_::TILE_BYTES;
  static constexpr int STAGE_OFF = 2 * B_::TILE_BYTES;
  static constexpr int STAGE = 2 * B_::TILE_BYTES + 2 * 512;
  static constexpr int BAR_OFF = STAGE_OFF + STG * STAGE;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;
  static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_P = 256, COL_DS = 320, COL_DV = 384, COL_DK = 448;
};

// dQ kernel shared memory: Q, dO; STG stages of (K, V).
template <int HD, int GROUP, int STG>
struct QCfg : BwdCfg<HD, GROUP> {
  using B_ = BwdCfg<HD, GROUP>;
  static constexpr int Q_OFF = 0, DO_OFF = B_::TILE_BYTES;
  static constexpr int STAGE_OFF = 2 * B_::TILE_BYTES;
  static constexpr int STAGE = 2 * B_::TILE_BYTES;
  static constexpr int BAR_OFF = STAGE_OFF + STG * STAGE;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;
  static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DS = 256, COL_DQ = 320;
};

// Barrier block (indices into uint64 slots).
// BB_S: S/dP of a tile in tensor memory; BB_SF: every compute warp has read
// them (the columns may take the next tile's); BB_P: P/dS (dS) written;
// BB_O: the gradient MMAs that read them have completed.
enum : int { BB_KV = 0, BB_S, BB_SF, BB_P, BB_O, BB_DONE, BB_STAGE0 };

// ------------------------------------------------------------ dK / dV
template <int HD, int GROUP, int STG>
__global__ void __launch_bounds__(BwdCfg<HD, GROUP>::THREADS, 1)
    swa_bwd_kv_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_do,
                      const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                      const SwaBwdParams p) {
  using Cfg = KvCfg<HD, GROUP, STG>;
  constexpr int TOK = Cfg::TOK;
  static_assert((BB_STAGE0 + 2 * STG) * 8 + 8 <= 256, "barrier block");
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::BAR_OFF);
  uint64_t* st_full = bars + BB_STAGE0;
  uint64_t* st_empty = st_full + STG;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(st_empty + STG);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // tile coordinates
  const int kt = blockIdx.x % p.ktiles;
  const int g = (blockIdx.x / p.ktiles) % p.Hkv;
  const int b = blockIdx.x / (p.ktiles * p.Hkv);
  const int64_t k0 = static_cast<int64_t>(kt) * 128;
  const int64_t q_end = (k0 + 127 + p.W < p.L) ? k0 + 127 + p.W : p.L;  // queries [k0, q_end)
  const int nq = static_cast<int>((q_end - k0 + TOK - 1) / TOK);

  if (threadIdx.x == 0) {
    mbar_init(&bars[BB_KV], 1);
    mbar_init(&bars[BB_S], 1);
    mbar_init(&bars[BB_P], Cfg::CWARPS);
    mbar_init(&bars[BB_SF], Cfg::CWARPS);
    mbar_init(&bars[BB_O], 1);
    mbar_init(&bars[BB_DONE], 1);
    for (int s = 0; s < STG; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == Cfg::WARP_MMA) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == Cfg::WARP_TMA) {
    // ================================================================ TMA
    if (lane == 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_do);
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      mbar_arrive_expect_tx(&bars[BB_KV], 2 * Cfg::TILE_BYTES);
      tma_load_4d(smem + Cfg::K_OFF, &map_k, &bars[BB_KV], 0, g, (int)k0, b);
      tma_load_4d(smem + Cfg::V_OFF, &map_v, &bars[BB_KV], 0, g, (int)k0, b);
      int issued = 0;
      for (int m = 0; m < nq; ++m) {
        const int s = m % STG;
        if (m >= STG && !mbar_wait(&st_empty[s], ((m / STG) - 1) & 1, abort_flag)) break;
        unsigned char* st = smem + Cfg::STAGE_OFF + s * Cfg::STAGE;
        const int64_t i0 = k0 + static_cast<int64_t>(m) * TOK;
        mbar_arrive_expect_tx(&st_full[s], 2 * Cfg::TILE_BYTES + 2 * 512);
        tma_load_4d(st, &map_q, &st_full[s], 0, g * GROUP, (int)i0, b);
        tma_load_4d(st + Cfg::TILE_BYTES, &map_do, &st_full[s], 0, g * GROUP, (int)i0, b);
        const int64_t off = ((static_cast<int64_t>(b) * p.Hkv + g) * p.Lp + i0) * GROUP;
        bulk_load(st + 2 * Cfg::TILE_BYTES, p.lse2s + off, 512, &st_full[s]);
        bulk_load(st + 2 * Cfg::TILE_BYTES + 512, p.Ds + off, 512, &st_full[s]);
        issued = m + 1;
      }
      // copies still in flight complete before the CTA can exit
      volatile int never = 0;
      mbar_wait(&bars[BB_KV], 0, &never);
      for (int m = (issued > STG ? issued - STG : 0); m < issued; ++m)
        mbar_wait(&st_full[m % STG], (m / STG) & 1, &never);
    }
  } else if (warp == Cfg::WARP_MMA) {
    // ================================================================ MMA
    constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, 0, 0);
    constexpr uint32_t IDESC_G = idesc_bf16_f32(128, HD, 0, 1);
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    const uint32_t base = smem_u32(smem);
    const uint64_t dK = smem_desc(base + Cfg::K_OFF, 16, Cfg::ATOM, Cfg::SWZ);
    const uint64_t dMN = smem_desc(base, 4096, Cfg::ATOM, Cfg::SWZ);  // MN-major B (N = HD = one atom row)
    const uint32_t hi_k = static_cast<uint32_t>(dK >> 32), hi_mn = static_cast<uint32_t>(dMN >> 32);
    const uint32_t lo_base = static_cast<uint32_t>(smem_desc(base, 16, Cfg::ATOM, Cfg::SWZ));
    const uint32_t lo_mn_base = static_cast<uint32_t>(dMN);
    auto d64 = [](uint32_t lo, uint32_t hi) { return (static_cast<uint64_t>(hi) << 32) | lo; };
    constexpr uint32_t kUnit = 16;  // descriptor address unit (bytes)
    auto stage_lo = [&](int s, int which) {  // K-major descriptor low word of the stage's Q (0) or dO (1)
      return lo_base + (Cfg::STAGE_OFF + s * Cfg::STAGE + which * Cfg::TILE_BYTES) / kUnit;
    };
    const uint32_t lo_k = lo_base + Cfg::K_OFF / kUnit, lo_v = lo_base + Cfg::V_OFF / kUnit;
    auto issue_sdp = [&](int s) {
      // Sᵀ = K Qᵀ and dPᵀ = V dOᵀ: M = 128 keys, N = 128 query rows, K = HD
      const uint32_t lq = stage_lo(s, 0), ldo = stage_lo(s, 1);
#pragma unroll
      for (int k = 0; k < HD / 16; ++k) {
        umma_ss_w(tmem + Cfg::COL_S, d64(lo_k + 2 * k, hi_k), d64(lq + 2 * k, hi_k), IDESC_S, k > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int k = 0; k < HD / 16; ++k) {
        umma_ss_w(tmem + Cfg::COL_DP, d64(lo_v + 2 * k, hi_k), d64(ldo + 2 * k, hi_k), IDESC_S, k > 0 ? 1u : 0u);
      }
    };
    auto issue_grad = [&](int s, bool first) {
      // dV += Pᵀ dO, dK += dSᵀ Q: M = 128 keys, N = HD, K = 128 query rows (16 per step)
      const uint32_t lq = lo_mn_base + (Cfg::STAGE_OFF + s * Cfg::STAGE) / kUnit;
      const uint32_t ldo = lq + Cfg::TILE_BYTES / kUnit;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        umma_ts_w(tmem + Cfg::COL_DV, tmem + Cfg::COL_P + 8 * k, d64(ldo + k * Cfg::ROW_BYTES, hi_mn), IDESC_G,
                  (first && k == 0) ? 0u : 1u);
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        umma_ts_w(tmem + Cfg::COL_DK, tmem + Cfg::COL_DS + 8 * k, d64(lq + k * Cfg::ROW_BYTES, hi_mn), IDESC_G,
                  (first && k == 0) ? 0u : 1u);
      }
    };
    // S/dP of tile m+1 go in as soon as the compute warps have read those of
    // tile m, so Sᵀ and dPᵀ run under tile m's exps; the gradient MMAs of
    // tile m follow once its P and dS are written.
    bool ok = wait(&bars[BB_KV], 0) && wait(&st_full[0], 0);
    if (ok) {
      tc_fence_after();
      issue_sdp(0);
      tc_commit_w(&bars[BB_S]);
    }
    for (int m = 0; m < nq && ok; ++m) {
      if (m + 1 < nq) {
        const int sn = (m + 1) % STG;
        ok = wait(&st_full[sn], ((m + 1) / STG) & 1) && wait(&bars[BB_SF], m & 1);
        if (!ok) break;
        tc_fence_after();
        issue_sdp(sn);
        tc_commit_w(&bars[BB_S]);
      }
      ok = wait(&bars[BB_P], m & 1);
      if (!ok) break;
      tc_fence_after();
      issue_grad(m % STG, m == 0);
      tc_commit_w(&bars[BB_O]);
      tc_commit_w(&st_empty[m % STG]);
    }
    tc_commit_w(&bars[BB_DONE]);
    volatile int never = 0;
    mbar_wait(&bars[BB_DONE], 0, &never);
  } else {
    // ============================================================ compute
    const int quarter = warp & 3, part = warp >> 2;
    const int r = quarter * 32 + lane;  // key row of the tile
    const int64_t j = k0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    bool ok = true;
    for (int m = 0; m < nq && ok; ++m) {
      const int s = m % STG;
      const int64_t i0 = k0 + static_cast<int64_t>(m) * TOK;
      ok = wait(&bars[BB_S], m & 1);
      // the stage's lse2 / D columns (written by the copy engine) are read below
      if (ok) ok = wait(&st_full[s], (m / STG) & 1);
      if (!ok) break;
      tc_fence_after();
      const float* lse2 = reinterpret_cast<const float*>(smem + Cfg::STAGE_OFF + s * Cfg::STAGE + 2 * Cfg::TILE_BYTES);
      const float* Dv = lse2 + 128;
      // the whole tile is inside the band when its first query sees the last
      // key and its last query still sees the first key
      const bool full = (i0 >= k0 + 127) && (i0 + TOK - 1 - k0 < p.W) && (i0 + TOK - 1 < p.L);
      // Key j sees the query tokens [j, min(j + W, L)): in this tile the
      // columns [clo, chi] (token (c / GROUP) + i0); an empty row gets an
      // interval no column falls in.  One unsigned compare per column.
      int clo = 0;
      unsigned cspan = 127u;
      if (!full) {
        const int64_t tlo = j > i0 ? j : i0;
        const int64_t thi_x = (j + p.W < p.L ? j + p.W : p.L);  // exclusive
        const int64_t thi = (thi_x < i0 + TOK ? thi_x : i0 + TOK) - 1;
        if (thi < tlo) {
          clo = 1 << 20;
          cspan = 0u;
        } else {
          clo = static_cast<int>(tlo - i0) * GROUP;
          cspan = static_cast<unsigned>((static_cast<int>(thi - i0) + 1) * GROUP - 1 - clo);
        }
      }
      {
        const int cc = part;  // this warp's 32 columns
        uint32_t sr[32], dr[32];
        tmem_ld32(tmem + lane_off + Cfg::COL_S + 32 * cc, sr);
        tmem_ld32(tmem + lane_off + Cfg::COL_DP + 32 * cc, dr);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[BB_SF]);  // the next tile's Sᵀ, dPᵀ may take these columns
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          float pv[2], dsv[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int c = 32 * cc + 2 * q + e;  // query row of the tile: token c / GROUP, head c % GROUP
            float pr = ex2b(fmaf(__uint_as_float(sr[2 * q + e]), p.scale_log2, -lse2[c]));
            pr = (static_cast<unsigned>(c - clo) <= cspan) ? pr : 0.f;
            pv[e] = pr;
            dsv[e] = pr * (__uint_as_float(dr[2 * q + e]) - Dv[c]);
          }
          pk[q] = pack_bf16x2(pv[0], pv[1]);
          dk[q] = pack_bf16x2(dsv[0], dsv[1]);
        }
        // P/dS of tile m-1 are read by its gradient MMAs until BB_O
        if (m > 0) {
          ok = wait(&bars[BB_O], (m - 1) & 1);
          if (!ok) break;
          tc_fence_after();
        }
        tmem_st16(tmem + lane_off + Cfg::COL_P + 16 * cc, pk);
        tmem_st16(tmem + lane_off + Cfg::COL_DS + 16 * cc, dk);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[BB_P]);
    }
    // ---- epilogue: dV, dK (· scale) -> bf16 rows of key j
    if (ok && nq > 0) ok = wait(&bars[BB_O], (nq - 1) & 1);
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t col = which == 0 ? Cfg::COL_DV : Cfg::COL_DK;
        const float mul = which == 0 ? 1.f : p.scale;
        __nv_bfloat16* dst = (which == 0 ? p.dv : p.dk) + ((static_cast<int64_t>(b) * p.L + j) * p.Hkv + g) * HD;
#pragma unroll
        for (int q = 0; q < HD / 16; ++q) {
          if (q % Cfg::NCW != part) continue;  // the parts of a quarter share the columns
          uint32_t t16[16];
          if (nq > 0) {
            tmem_ld16(tmem + lane_off + col + 16 * q, t16);
            tc_wait_ld();
          } else {
#pragma unroll
            for (int c = 0; c < 16; ++c) t16[c] = 0u;
          }
          if (j < p.L && SAMBA_CHECK(j >= 0 && b < p.B && g < p.Hkv)) {
            uint4 v0, v1;
            v0.x = pack_bf16x2(__uint_as_float(t16[0]) * mul, __uint_as_float(t16[1]) * mul);
            v0.y = pack_bf16x2(__uint_as_float(t16[2]) * mul, __uint_as_float(t16[3]) * mul);
            v0.z = pack_bf16x2(__uint_as_float(t16[4]) * mul, __uint_as_float(t16[5]) * mul);
            v0.w = pack_bf16x2(__uint_as_float(t16[6]) * mul, __uint_as_float(t16[7]) * mul);
            v1.x = pack_bf16x2(__uint_as_float(t16[8]) * mul, __uint_as_float(t16[9]) * mul);
            v1.y = pack_bf16x2(__uint_as_float(t16[10]) * mul, __uint_as_float(t16[11]) * mul);
            v1.z = pack_bf16x2(__uint_as_float(t16[12]) * mul, __uint_as_float(t16[13]) * mul);
            v1.w = pack_bf16x2(__uint_as_float(t16[14]) * mul, __uint_as_float(t16[15]) * mul);
            reinterpret_cast<uint4*>(dst + 16 * q)[0] = v0;
            reinterpret_cast<uint4*>(dst + 16 * q)[1] = v1;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == Cfg::WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ----------------------------------------------------------------- dQ
template <int HD, int GROUP, int STG>
__global__ void __launch_bounds__(BwdCfg<HD, GROUP>::THREADS, 1)
    swa_bwd_q_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_do,
                     const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                     const SwaBwdParams p) {
  using Cfg = QCfg<HD, GROUP, STG>;
  constexpr int TOK = Cfg::TOK;
  static_assert((BB_STAGE0 + 2 * STG) * 8 + 8 <= 256, "barrier block");
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::BAR_OFF);
  uint64_t* st_full = bars + BB_STAGE0;
  uint64_t* st_empty = st_full + STG;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(st_empty + STG);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int qt = blockIdx.x % p.qtiles;
  const int g = (blockIdx.x / p.qtiles) % p.Hkv;
  const int b = blockIdx.x / (p.qtiles * p.Hkv);
  const int64_t i0 = static_cast<int64_t>(qt) * TOK;
  const int64_t top = i0 + TOK;  // key tiles aligned to the top of the query tile
  const int64_t n_band = (p.W + TOK - 1 + 127) / 128, n_pos = (top + 127) / 128;
  const int nt = static_cast<int>(n_band < n_pos ? n_band : n_pos);

  if (threadIdx.x == 0) {
    mbar_init(&bars[BB_KV], 1);  // here: Q and dO landed
    mbar_init(&bars[BB_S], 1);
    mbar_init(&bars[BB_P], Cfg::CWARPS);
    mbar_init(&bars[BB_SF], Cfg::CWARPS);
    mbar_init(&bars[BB_O], 1);
    mbar_init(&bars[BB_DONE], 1);
    for (int s = 0; s < STG; ++s) {
      mbar_init(&st_full[s], 1);
      mbar_init(&st_empty[s], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == Cfg::WARP_MMA) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == Cfg::WARP_TMA) {
    // ================================================================ TMA
    if (lane == 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_do);
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      mbar_arrive_expect_tx(&bars[BB_KV], 2 * Cfg::TILE_BYTES);
      tma_load_4d(smem + Cfg::Q_OFF, &map_q, &bars[BB_KV], 0, g * GROUP, (int)i0, b);
      tma_load_4d(smem + Cfg::DO_OFF, &map_do, &bars[BB_KV], 0, g * GROUP, (int)i0, b);
      int issued = 0;
      for (int t = 0; t < nt; ++t) {
        const int s = t % STG;
        if (t >= STG && !mbar_wait(&st_empty[s], ((t / STG) - 1) & 1, abort_flag)) break;
        unsigned char* st = smem + Cfg::STAGE_OFF + s * Cfg::STAGE;
        const int kk0 = (int)(top - 128 * (t + 1));
        mbar_arrive_expect_tx(&st_full[s], 2 * Cfg::TILE_BYTES);
        tma_load_4d(st, &map_k, &st_full[s], 0, g, kk0, b);
        tma_load_4d(st + Cfg::TILE_BYTES, &map_v, &st_full[s], 0, g, kk0, b);
        issued = t + 1;
      }
      volatile int never = 0;
      mbar_wait(&bars[BB_KV], 0, &never);
      for (int t = (issued > STG ? issued - STG : 0); t < issued; ++t)
        mbar_wait(&st_full[t % STG], (t / STG) & 1, &never);
    }
  } else if (warp == Cfg::WARP_MMA) {
    // ================================================================ MMA
    constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, 0, 0);
    constexpr uint32_t IDESC_G = idesc_bf16_f32(128, HD, 0, 1);
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    const uint32_t base = smem_u32(smem);
    const uint64_t dKm = smem_desc(base, 16, Cfg::ATOM, Cfg::SWZ);
    const uint64_t dMN = smem_desc(base, 4096, Cfg::ATOM, Cfg::SWZ);
    const uint32_t hi_k = static_cast<uint32_t>(dKm >> 32), hi_mn = static_cast<uint32_t>(dMN >> 32);
    const uint32_t lo_base = static_cast<uint32_t>(dKm), lo_mn_base = static_cast<uint32_t>(dMN);
    auto d64 = [](uint32_t lo, uint32_t hi) { return (static_cast<uint64_t>(hi) << 32) | lo; };
    constexpr uint32_t kUnit = 16;
    const uint32_t lo_q = lo_base + Cfg::Q_OFF / kUnit, lo_do = lo_base + Cfg::DO_OFF / kUnit;
    auto issue_sdp = [&](int s) {
      // S = Q Kᵀ and dP = dO Vᵀ: M = 128 query rows, N = 128 keys, K = HD
      const uint32_t lk = lo_base + (Cfg::STAGE_OFF + s * Cfg::STAGE) / kUnit;
      const uint32_t lv = lk + Cfg::TILE_BYTES / kUnit;
#pragma unroll
      for (int k = 0; k < HD / 16; ++k)
        umma_ss_w(tmem + Cfg::COL_S, d64(lo_q + 2 * k, hi_k), d64(lk + 2 * k, hi_k), IDESC_S, k > 0 ? 1u : 0u);
#pragma unroll
      for (int k = 0; k < HD / 16; ++k)
        umma_ss_w(tmem + Cfg::COL_DP, d64(lo_do + 2 * k, hi_k), d64(lv + 2 * k, hi_k), IDESC_S, k > 0 ? 1u : 0u);
    };
    auto issue_dq = [&](int s, bool first) {
      // dQ += dS K: M = 128 query rows, N = HD, K = 128 keys (16 per step), K tile MN-major
      const uint32_t lk = lo_mn_base + (Cfg::STAGE_OFF + s * Cfg::STAGE) / kUnit;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        umma_ts_w(tmem + Cfg::COL_DQ, tmem + Cfg::COL_DS + 8 * k, d64(lk + k * Cfg::ROW_BYTES, hi_mn), IDESC_G,
                  (first && k == 0) ? 0u : 1u);
    };
    // S/dP of key tile t+1 go in as soon as the compute warps have read
    // those of tile t; dQ of tile t follows once its dS is written.
    bool ok = wait(&bars[BB_KV], 0) && wait(&st_full[0], 0);
    if (ok) {
      tc_fence_after();
      issue_sdp(0);
      tc_commit_w(&bars[BB_S]);
    }
    for (int t = 0; t < nt && ok; ++t) {
      if (t + 1 < nt) {
        const int sn = (t + 1) % STG;
        ok = wait(&st_full[sn], ((t + 1) / STG) & 1) && wait(&bars[BB_SF], t & 1);
        if (!ok) break;
        tc_fence_after();
        issue_sdp(sn);
        tc_commit_w(&bars[BB_S]);
      }
      ok = wait(&bars[BB_P], t & 1);
      if (!ok) break;
      tc_fence_after();
      issue_dq(t % STG, t == 0);
      tc_commit_w(&bars[BB_O]);
      tc_commit_w(&st_empty[t % STG]);
    }
    tc_commit_w(&bars[BB_DONE]);
    volatile int never = 0;
    mbar_wait(&bars[BB_DONE], 0, &never);
  } else {
    // ============================================================ compute
    const int quarter = warp & 3, part = warp >> 2;
    const int r = quarter * 32 + lane;  // query row: token r / GROUP, head r % GROUP
    const int tok = r / GROUP, hh = r % GROUP;
    const int64_t irow = i0 + tok;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int64_t rix = ((static_cast<int64_t>(b) * p.Hkv + g) * p.Lp + i0) * GROUP + r;
    const float lse2 = p.lse2s[rix], Dr = p.Ds[rix];
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    bool ok = true;
    for (int t = 0; t < nt && ok; ++t) {
      const int64_t kk0 = top - 128 * (t + 1);
      ok = wait(&bars[BB_S], t & 1);
      if (!ok) break;
      tc_fence_after();
      const bool full = (kk0 + 127 <= i0) && (i0 + TOK - 1 - kk0 < p.W) && (kk0 >= 0) && (i0 + TOK - 1 < p.L);
      // Row irow sees the keys [max(0, irow - W + 1), irow] (none past L):
      // the columns [clo, clo + cspan] of this key tile.
      int clo = 0;
      unsigned cspan = 127u;
      if (!full) {
        const int64_t jlo = irow - p.W + 1 > 0 ? irow - p.W + 1 : 0;
        const int64_t lo = jlo - kk0 > 0 ? jlo - kk0 : 0;
        const int64_t hi = irow - kk0 < 127 ? irow - kk0 : 127;
        if (irow >= p.L || hi < lo) {
          clo = 1 << 20;
          cspan = 0u;
        } else {
          clo = static_cast<int>(lo);
          cspan = static_cast<unsigned>(hi - lo);
        }
      }
      {
        const int cc = part;  // this warp's 32 columns
        uint32_t sr[32], dr[32];
        tmem_ld32(tmem + lane_off + Cfg::COL_S + 32 * cc, sr);
        tmem_ld32(tmem + lane_off + Cfg::COL_DP + 32 * cc, dr);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[BB_SF]);  // the next key tile's S, dP may take these columns
        uint32_t dk[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          float dsv[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int c = 32 * cc + 2 * q + e;
            float pr = ex2b(fmaf(__uint_as_float(sr[2 * q + e]), p.scale_log2, -lse2));
            pr = (static_cast<unsigned>(c - clo) <= cspan) ? pr : 0.f;
            dsv[e] = pr * (__uint_as_float(dr[2 * q + e]) - Dr);
          }
          dk[q] = pack_bf16x2(dsv[0], dsv[1]);
        }
        // dS of key tile t-1 is read by its dQ MMAs until BB_O
        if (t > 0) {
          ok = wait(&bars[BB_O], (t - 1) & 1);
          if (!ok) break;
          tc_fence_after();
        }
        tmem_st16(tmem + lane_off + Cfg::COL_DS + 16 * cc, dk);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[BB_P]);
    }
    if (ok && nt > 0) ok = wait(&bars[BB_O], (nt - 1) & 1);
    // The tensor-memory loads are warp-collective: every lane of the warp
    // takes them (ok is warp-uniform); only the stores depend on the row.
    if (ok) {
      tc_fence_after();
      __nv_bfloat16* dst = p.dq + ((static_cast<int64_t>(b) * p.L + irow) * p.Hq + g * GROUP + hh) * HD;
#pragma unroll
      for (int q = 0; q < HD / 16; ++q) {
        if (q % Cfg::NCW != part) continue;  // the parts of a quarter share the columns
        uint32_t t16[16];
        tmem_ld16(tmem + lane_off + Cfg::COL_DQ + 16 * q, t16);
        tc_wait_ld();
        if (irow >= p.L || !SAMBA_CHECK(irow >= 0 && b < p.B && g * GROUP + hh < p.Hq)) continue;
        uint4 v0, v1;
        const float mul = p.scale;
        v0.x = pack_bf16x2(__uint_as_float(t16[0]) * mul, __uint_as_float(t16[1]) * mul);
        v0.y = pack_bf16x2(__uint_as_float(t16[2]) * mul, __uint_as_float(t16[3]) * mul);
        v0.z = pack_bf16x2(__uint_as_float(t16[4]) * mul, __uint_as_float(t16[5]) * mul);
        v0.w = pack_bf16x2(__uint_as_float(t16[6]) * mul, __uint_as_float(t16[7]) * mul);
        v1.x = pack_bf16x2(__uint_as_float(t16[8]) * mul, __uint_as_float(t16[9]) * mul);
        v1.y = pack_bf16x2(__uint_as_float(t16[10]) * mul, __uint_as_float(t16[11]) * mul);
        v1.z = pack_bf16x2(__uint_as_float(t16[12]) * mul, __uint_as_float(t16[13]) * mul);
        v1.w = pack_bf16x2(__uint_as_float(t16[14]) * mul, __uint_as_float(t16[15]) * mul);
        reinterpret_cast<uint4*>(dst + 16 * q)[0] = v0;
        reinterpret_cast<uint4*>(dst + 16 * q)[1] = v1;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == Cfg::WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

constexpr int kKvStages = 3, kQStages = 4;
// Each CTA allocates all 512 tensor-memory columns, so no two may share an SM
// (a second allocation would wait for the first CTA to finish): the launch
// asks for more than half of an SM's shared memory.
constexpr int kOneCtaSmem = 120 * 1024;

template <int HD, int GROUP>
int launch_swa_bwd_t(const samba_swa_bwd_args& a, cudaStream_t stream) {
  using KC = KvCfg<HD, GROUP, kKvStages>;
  using QC = QCfg<HD, GROUP, kQStages>;
  auto kkv = swa_bwd_kv_kernel<HD, GROUP, kKvStages>;
  auto kq = swa_bwd_q_kernel<HD, GROUP, kQStages>;
  const int smem_kv = std::max(KC::SMEM, kOneCtaSmem), smem_q = std::max(QC::SMEM, kOneCtaSmem);
  static PerDeviceOnce attr;
  const int arc = once_per_device(attr, [&] {
    return (cudaFuncSetAttribute(kkv, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_kv) == cudaSuccess &&
            cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_q) == cudaSuccess)
               ? SAMBA_OK
               : fail(SAMBA_ERR_CUDA, "samba_swa_bwd: cannot set shared memory size");
  });
  if (arc != SAMBA_OK) return arc;
  const uint64_t B = a.batch, L = a.seqlen, Hq = a.heads_q, Hkv = a.heads_kv;
  const CUtensorMapSwizzle swz =
      HD == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : (HD == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  CUtensorMap mq, mdo, mk, mv;
  {
    const uint64_t dq[4] = {(uint64_t)HD, Hq, L, B};
    const uint64_t sq[3] = {HD * 2ull, Hq * HD * 2ull, L * Hq * HD * 2ull};
    const uint32_t bq[4] = {(uint32_t)HD, (uint32_t)GROUP, (uint32_t)KC::TOK, 1};
    int rc = encode_tiled(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.q, dq, sq, bq, swz, "swa bwd q");
    if (rc) return rc;
    rc = encode_tiled(&mdo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.dO, dq, sq, bq, swz, "swa bwd dO");
    if (rc) return rc;
    const uint64_t dk[4] = {(uint64_t)HD, Hkv, L, B};
    const uint64_t sk[3] = {HD * 2ull, Hkv * HD * 2ull, L * Hkv * HD * 2ull};
    const uint32_t bk[4] = {(uint32_t)HD, 1, 128, 1};
    rc = encode_tiled(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.k, dk, sk, bk, swz, "swa bwd k");
    if (rc) return rc;
    rc = encode_tiled(&mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.v, dk, sk, bk, swz, "swa bwd v");
    if (rc) return rc;
  }
  SwaBwdParams p;
  p.o = reinterpret_cast<const __nv_bfloat16*>(a.o);
  p.dO = reinterpret_cast<const __nv_bfloat16*>(a.dO);
  p.lse = a.lse;
  p.L = a.seqlen;
  p.Lp = (a.seqlen + 127) / 128 * 128;
  p.W = a.window;
  p.Hq = a.heads_q;
  p.Hkv = a.heads_kv;
  p.B = (int)a.batch;
  p.lse2s = reinterpret_cast<float*>(a.workspace);
  p.Ds = p.lse2s + static_cast<int64_t>(a.batch) * a.heads_q * p.Lp;
  p.dq = reinterpret_cast<__nv_bfloat16*>(a.dq);
  p.dk = reinterpret_cast<__nv_bfloat16*>(a.dk);
  p.dv = reinterpret_cast<__nv_bfloat16*>(a.dv);
  p.scale = a.scale > 0.f ? a.scale : 1.0f / std::sqrt((float)HD);
  p.scale_log2 = p.scale * kLog2eB;
  p.ktiles = (int)((a.seqlen + 127) / 128);
  p.qtiles = (int)((a.seqlen + KC::TOK - 1) / KC::TOK);
  const int64_t nkv = (int64_t)p.ktiles * a.heads_kv * a.batch, nq = (int64_t)p.qtiles * a.heads_kv * a.batch;
  if (nkv > INT32_MAX || nq > INT32_MAX) return fail(SAMBA_ERR_UNSUPPORTED, "samba_swa_bwd: problem too large");
  {
    const int64_t n = (int64_t)a.batch * p.Lp * a.heads_q;
    const int64_t blocks = std::min<int64_t>((n + 255) / 256, int64_t(sm_count()) * 16);
    swa_bwd_prep_kernel<HD><<<(unsigned)blocks, 256, 0, stream>>>(p, GROUP);
    int rc = check_launch("samba_swa_bwd (prep)");
    if (rc) return rc;
  }
  kkv<<<(unsigned)nkv, KC::THREADS, smem_kv, stream>>>(mq, mdo, mk, mv, p);
  int rc = check_launch("samba_swa_bwd (dk, dv)");
  if (rc) return rc;
  kq<<<(unsigned)nq, QC::THREADS, smem_q, stream>>>(mq, mdo, mk, mv, p);
  return check_launch("samba_swa_bwd (dq)");
}

template <int HD>
int launch_swa_bwd_hd(const samba_swa_bwd_args& a, cudaStream_t s) {
  switch (a.heads_q / a.heads_kv) {
    case 1: return launch_swa_bwd_t<HD, 1>(a, s);
    case 2: return launch_swa_bwd_t<HD, 2>(a, s);
    case 4: return launch_swa_bwd_t<HD, 4>(a, s);
    case 8: return launch_swa_bwd_t<HD, 8>(a, s);
    default: return launch_swa_bwd_t<HD, 16>(a, s);
  }
}

}  // namespace

size_t swa_bwd_workspace(int64_t B, int64_t L, int Hq) {
  const int64_t Lp = (L + 127) / 128 * 128;
  size_t r = 0;
  if (__builtin_mul_overflow(static_cast<size_t>(B), static_cast<size_t>(Lp), &r) ||
      __builtin_mul_overflow(r, static_cast<size_t>(Hq), &r) || __builtin_mul_overflow(r, 2 * sizeof(float), &r))
    return SIZE_MAX;
  return r;
}

int launch_swa_bwd(const samba_swa_bwd_args& a, cudaStream_t s) {
  switch (a.head_dim) {
    case 16: return launch_swa_bwd_hd<16>(a, s);
    case 32: return launch_swa_bwd_hd<32>(a, s);
    default: return launch_swa_bwd_hd<64>(a, s);
  }
}

}  // namespace samba
