// Backward of the fused selective-scan prefill: the gradients of y with
// respect to x, delta, A, B, C, D, z, the conv weights and bias, h0 and the
// conv state.
//
// Page "SAMBA混合注意力状态空间模型", section 数学框架 / Mamba层: the
// recurrence h_t = Ā_t h_{t-1} + B̄_t x_t, y_t = C_t h_t with input-dependent
// B, C and Δ (readings as in the forward: Ā = exp(ΔA), B̄x = ΔBu, u the conv
// + SiLU output, Δ = softplus(delta), y gated by silu(z) with a D skip).
// Reverse mode walks the recurrence backwards: with G_t = ∂L/∂h_t,
//   G_t = C_t g_t + Ā_{t+1} G_{t+1},   g_t = dy_t silu(z_t),
//   dC_t = Σ_c g_t h_t,  dB_t = Σ_c G_t Δ_t u_t,  dA = Σ_t G_t Δ_t Ā_t h_{t-1},
//   dΔ_t = Σ_n G_t (A Ā_t h_{t-1} + B_t u_t),  du_t = D g_t + Δ_t Σ_n G_t B_t,
// then through softplus, the conv's SiLU and the conv itself.
//
// Design: one CTA per (sequence b, 32 channels), 4 warps; lane = channel and
// warp w holds states [w·N/4, (w+1)·N/4) of every channel, as the forward's
// scan warps do.  The walk needs h_{t-1} in reverse order, so it is
// recomputed: a first pass runs the recurrence forward over the whole
// sequence and stores the state at the start of every 16-token chunk in the
// workspace (or the forward kernel has stored them, and the pass is
// skipped); the reverse pass then takes the chunks last to first, recomputes
// the chunk's 16 states into shared memory from its checkpoint, and walks it
// backwards.  Per chunk, all 128 threads share the per-(token, channel) work
// (conv, softplus, gate, and their gradients) with thread = (channel, token
// mod 4).  dB and dC sum over the channels of the whole layer: each warp
// reduces its lanes (a transposing butterfly: 2·N/4 sums in 9 shuffles at
// N = 16), the CTA collects the chunk's [16 tokens × N] sums in shared memory
// and writes them as one contiguous row block of its own partial in the
// workspace, and a second kernel adds the partials of all channel blocks
// (no atomics on these: every element would take one from each of the D/32
// blocks).  dA, dD and the conv gradients sum over tokens in registers and
// over the batch with atomics at the end, into outputs the launcher clears.
// No waits other than __syncthreads.
#include "common.cuh"
#include "host.hpp"

namespace samba {

#ifndef SAMBA_SCAN_BWD_CTAS
#define SAMBA_SCAN_BWD_CTAS 4  // CTAs per SM the launch bounds aim at
#endif

namespace {

constexpr int kCh = 32;      // channels per CTA (one per lane)
constexpr int kTc = 16;      // tokens per chunk
// Warps per CTA: one per group of N / warps states (8 warps of 2 states at
// N = 16); with 56 KB of shared memory and at most 64 registers a thread at
// N = 16, every SM holds four CTAs of 8 warps.
constexpr int nwarps(int N) { return N >= 8 ? 8 : 4; }
constexpr int kHalo = 3;     // earlier inputs the conv needs (K <= 4)
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float sigmoid_dev(float v) { return __fdividef(1.0f, 1.0f + __expf(-v)); }
__device__ __forceinline__ float softplus_b(float w) {
  return w > 20.0f ? w : (w > 0.0f ? w + log1pf(__expf(-w)) : log1pf(__expf(w)));
}

template <typename T>
__device__ __forceinline__ float ldv(const T* p, int64_t i) {
  return to_f32<T>(p[i]);
}
template <typename T>
__device__ __forceinline__ void stv(void* p, int64_t i, float v) {
  reinterpret_cast<T*>(p)[i] = from_f32<T>(v);
}

// One halving exchange of warp_sum_many: lanes with `bit` set keep values
// [H, 2H) and the others [0, H), each adding its partner's copy.
template <int H>
__device__ __forceinline__ void halve(float* a, bool upper, int bit) {
#pragma unroll
  for (int i = 0; i < H; ++i) {
    const float send = upper ? a[i] : a[i + H];
    const float keep = upper ? a[i + H] : a[i];
    a[i] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
  }
}

// log2(M) halving exchanges over lane bits BIT, BIT/2, ...: afterwards a[0]
// holds one of the M values summed over the M lanes that differ in those
// bits; idx gets its index, most significant bit first.
template <int M, int BIT>
__device__ __forceinline__ void halving(float* a, int lane, int& idx) {
  if constexpr (M > 1) {
    const bool up = (lane & BIT) != 0;
    halve<M / 2>(a, up, BIT);
    idx = idx * 2 + (up ? 1 : 0);
    halving<M / 2, BIT / 2>(a, lane, idx);
  }
}
template <int BIT>
__device__ __forceinline__ float finish_sum(float s) {
  if constexpr (BIT >= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, BIT);
    return finish_sum<BIT / 2>(s);
  } else {
    return s;
  }
}
constexpr int ilog2(int m) { return m <= 1 ? 0 : 1 + ilog2(m / 2); }

// Sums each of the M values a[0..M) (M a power of two, 2..32) over the 32
// lanes of the warp with M - 1 + (5 - log2 M) shuffles instead of 5·M.
// Returns the total of value *which; the 32 / M lanes that agree in their
// top log2(M) bits hold the same value.
template <int M>
__device__ __forceinline__ float warp_sum_many(float (&a)[M], int lane, int* which) {
  static_assert(M == 2 || M == 4 || M == 8 || M == 16 || M == 32, "M");
  int idx = 0;
  halving<M, 16>(a, lane, idx);
  *which = idx;
  return finish_sum<(16 >> ilog2(M))>(a[0]);
}

struct ScanBwdParams {
  const void* x;
  const float* delta;
  const float* A;
  const float* Bm;
  const float* Cm;
  const float* Dskip;
  const void* z;
  const float* conv_w;
  const float* conv_b;
  const float* h0;
  const float* conv_state_in;
  const void* dy;
  void* dx;
  float* ddelta;
  void* dz;
  float* dA;
  float* dB;
  float* dC;
  float* dD;
  float* dconv_w;
  float* dconv_b;
  float* dh0;
  float* dconv_state;
  float* ckpt;  // [B, nchunks, N, D]: the workspace's, or the forward's
  bool ckpt_given;  // the forward wrote ckpt: no first pass
  float* part;  // [D/32 blocks][2 (dB, dC)][B, L, N]
  int64_t L, D;
  int K;
  int nchunks;
  uint32_t flags;
};

template <int N>
struct ScanBwdSmem {
  float x[kTc + kHalo][kCh];   // inputs of the chunk and the 3 before it
  float u[kTc][kCh];
  float dt[kTc][kCh];
  float sg[kTc][kCh];          // σ(delta): d softplus / d delta
  float gy[kTc][kCh];          // dy · silu(z)
  float dydsz[kTc][kCh];       // dy · silu'(z)
  float Bv[kTc][N];
  float Cv[kTc][N];
  union {
    float H[kTc][N][kCh];      // h_t of the chunk (during the chunks)
    float red[3 + 4][nwarps(N)][kCh];  // per-channel sums of the token lanes (dD, dconv_b, dconv_w[K]; at the end)
  };
  float part[2][kTc][kCh];     // sums over the warps' states: [0] C·h (forward) / dΔ (reverse), [1] du
  float dc[kTc + kHalo][kCh];  // conv-output gradient, rows kTc.. = first rows of the later chunk
  float dbc[2][kTc][N];        // this block's dB, dC of the chunk (summed over its channels)
};

// Global inputs of one chunk for one thread, fetched a chunk ahead into
// registers so that their latency hides behind the work on the chunk before.
template <int N>
struct ChunkRegs {
  static constexpr int NW = nwarps(N), kThreads = 32 * NW;
  static constexpr int XR = (kTc + kHalo + NW - 1) / NW, TR = kTc / NW;
  static constexpr int kBC = (kTc * N + kThreads - 1) / kThreads;
  float x[XR];       // rows pt, pt+NW, ... of [3 earlier tokens ; the chunk]
  float delta[TR], z[TR], dy[TR];
  float Bv[kBC], Cv[kBC];
};

template <int N, typename XT, typename YT>
__global__ void __launch_bounds__(32 * nwarps(N), SAMBA_SCAN_BWD_CTAS) scan_bwd_kernel(const ScanBwdParams p) {
  constexpr int NW = nwarps(N);
  constexpr int kThreads = 32 * NW;
  constexpr int SPL = N / NW;  // states per lane
  using CR = ChunkRegs<N>;
  constexpr int G4 = 4;        // tokens per reduction group
  constexpr int NV = G4 * 2 * SPL;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ScanBwdSmem<N>& S = *reinterpret_cast<ScanBwdSmem<N>*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t b = blockIdx.y;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kCh;
  const int64_t D = p.D, L = p.L;
  const int K = p.K;
  const bool fuse = (p.flags & SAMBA_SCAN_FUSE_CONV) != 0;
  const bool csilu = (p.flags & SAMBA_SCAN_CONV_SILU) != 0;
  const bool splus = (p.flags & SAMBA_SCAN_DELTA_SOFTPLUS) != 0;
  const XT* x = reinterpret_cast<const XT*>(p.x);
  const XT* z = reinterpret_cast<const XT*>(p.z);
  const YT* dyp = reinterpret_cast<const YT*>(p.dy);

  // scan roles: lane = channel, warp = group of SPL states
  const int64_t ch_l = c0 + lane;
  const bool lane_ok = ch_l < D;
  float Al[SPL];
#pragma unroll
  for (int j = 0; j < SPL; ++j) Al[j] = lane_ok ? p.A[ch_l * N + warp * SPL + j] * kLog2e : 0.f;

  // token-parallel roles: thread = (channel pc, token lane pt)
  const int pc = lane, pt = warp;
  const int64_t ch_p = c0 + pc;
  const bool ch_ok = ch_p < D;
  float cw[4] = {0.f, 0.f, 0.f, 0.f}, cb = 0.f, dsk = 0.f;
  if (ch_ok) {
    if (fuse) {
      #pragma unroll
      for (int k = 0; k < 4; ++k)
        if (k < K) cw[k] = p.conv_w[ch_p * K + k];
      if (p.conv_b) cb = p.conv_b[ch_p];
    }
    if (p.Dskip) dsk = p.Dskip[ch_p];
  }
  auto chunk_len = [&](int c) {
    const int64_t rem = L - static_cast<int64_t>(c) * kTc;
    return static_cast<int>(rem < kTc ? rem : kTc);
  };

  // ---- the chunk's global inputs into registers (`full`: also z, dy, C)
  auto fetch = [&](int c, bool full, ChunkRegs<N>& R) {
    const int64_t t0 = static_cast<int64_t>(c) * kTc;
    const int nv = chunk_len(c);
#pragma unroll
    for (int i = 0; i < CR::XR; ++i) {
      const int r = pt + NW * i;
      const int64_t tau = t0 - kHalo + r;
      float v = 0.f;
      if (r < kTc + kHalo && ch_ok) {
        if (tau >= 0) {
          if (r - kHalo < nv) v = ldv<XT>(x, (b * L + tau) * D + ch_p);
        } else if (fuse && p.conv_state_in) {
          const int64_t pidx = tau + (K - 1);  // index into [conv state ; x]
          if (pidx >= 0) v = p.conv_state_in[(b * D + ch_p) * (K - 1) + pidx];
        }
      }
      R.x[i] = v;
    }
#pragma unroll
    for (int i = 0; i < CR::TR; ++i) {
      const int t = pt + NW * i;
      const bool ok = ch_ok && t < nv;
      const int64_t e = (b * L + t0 + t) * D + ch_p;
      R.delta[i] = ok ? p.delta[e] : 0.f;
      R.z[i] = (ok && full && z) ? ldv<XT>(z, e) : 0.f;
      R.dy[i] = (ok && full) ? ldv<YT>(dyp, e) : 0.f;
    }
#pragma unroll
    for (int i = 0; i < ChunkRegs<N>::kBC; ++i) {
      const int e = tid + kThreads * i;
      const int t = e / N;
      const bool ok = e < kTc * N && t < nv;
      R.Bv[i] = ok ? p.Bm[(b * L + t0) * N + e] : 0.f;
      R.Cv[i] = (ok && full) ? p.Cm[(b * L + t0) * N + e] : 0.f;
    }
  };

  // ---- registers -> shared memory, and the token-parallel prologue
  auto stage = [&](int c, bool full, const ChunkRegs<N>& R) {
    const int nv = chunk_len(c);
#pragma unroll
    for (int i = 0; i < CR::XR; ++i) {
      const int r = pt + NW * i;
      if (r < kTc + kHalo) S.x[r][pc] = R.x[i];
    }
#pragma unroll
    for (int i = 0; i < ChunkRegs<N>::kBC; ++i) {
      const int e = tid + kThreads * i;
      if (e < kTc * N) {
        S.Bv[e / N][e % N] = R.Bv[i];
        if (full) S.Cv[e / N][e % N] = R.Cv[i];
      }
    }
    __syncthreads();  // the conv below reads rows that other warps stored
#pragma unroll
    for (int i = 0; i < CR::TR; ++i) {
      const int t = pt + NW * i;
      const bool ok = ch_ok && t < nv;
      S.part[0][t][pc] = 0.f;  // the sums the warps add into start from zero
      S.part[1][t][pc] = 0.f;
      float u = 0.f, pre = 0.f, dt = 0.f, sg = 0.f;
      if (ok) {
        if (fuse) {
          pre = cb;
          #pragma unroll
          for (int k = 0; k < 4; ++k)
            if (k < K) pre = fmaf(cw[k], S.x[t + kHalo - (K - 1) + k][pc], pre);
          u = csilu ? __fdividef(pre, 1.0f + __expf(-pre)) : pre;
        } else {
          u = S.x[t + kHalo][pc];
        }
        const float w = R.delta[i];
        dt = splus ? softplus_b(w) : w;
        if (full) sg = splus ? sigmoid_dev(w) : 1.f;
      }
      S.u[t][pc] = u;
      S.dt[t][pc] = dt;
      if (full) {
        S.sg[t][pc] = sg;
        float gyv = 0.f, dszv = 0.f;
        if (ok) {
          gyv = R.dy[i];
          if (z) {
            const float zv = R.z[i];
            const float sgz = sigmoid_dev(zv);
            gyv = R.dy[i] * (zv * sgz);
            dszv = R.dy[i] * (sgz * (1.f + zv * (1.f - sgz)));
          }
        }
        S.gy[t][pc] = gyv;
        S.dydsz[t][pc] = dszv;
      }
    }
    __syncthreads();
  };

  ChunkRegs<N> R;

  // ------------------------------------------------ pass 1: checkpoints
  float h[SPL];
#pragma unroll
  for (int j = 0; j < SPL; ++j) h[j] = (p.h0 && lane_ok) ? p.h0[(b * D + ch_l) * N + warp * SPL + j] : 0.f;
  if (!p.ckpt_given) fetch(0, false, R);
  for (int c = 0; c < (p.ckpt_given ? 0 : p.nchunks); ++c) {
    const int nv = chunk_len(c);
    stage(c, false, R);
    if (c + 1 < p.nchunks) fetch(c + 1, false, R);
    if (lane_ok) {
#pragma unroll
      for (int j = 0; j < SPL; ++j) p.ckpt[((b * p.nchunks + c) * N + warp * SPL + j) * D + ch_l] = h[j];
    }
    // All kTc tokens, unrolled: past nv the staged Δ and u are zero, so
    // those steps leave h unchanged (exp(0) = 1, no input).
#pragma unroll
    for (int t = 0; t < kTc; ++t) {
      const float dt = S.dt[t][lane], du = dt * S.u[t][lane];
#pragma unroll
      for (int j = 0; j < SPL; ++j) h[j] = fmaf(ex2_fast(dt * Al[j]), h[j], du * S.Bv[t][warp * SPL + j]);
    }
    __syncthreads();
  }

  // ------------------------------------------------ pass 2: reverse walk
  float g[SPL], dAacc[SPL];
#pragma unroll
  for (int j = 0; j < SPL; ++j) g[j] = dAacc[j] = 0.f;
  float accD = 0.f, accB = 0.f, accW[4] = {0.f, 0.f, 0.f, 0.f};
  for (int r = pt; r < kHalo; r += NW) S.dc[kTc + r][pc] = 0.f;  // nothing after the last token
  // the checkpoint a chunk starts from is fetched with its inputs, a chunk ahead
  auto fetch_ckpt = [&](int c, float (&dst)[SPL]) {
#pragma unroll
    for (int j = 0; j < SPL; ++j) dst[j] = lane_ok ? p.ckpt[((b * p.nchunks + c) * N + warp * SPL + j) * D + ch_l] : 0.f;
  };
  float hs_next[SPL];
  fetch(p.nchunks - 1, true, R);
  fetch_ckpt(p.nchunks - 1, hs_next);
  for (int c = p.nchunks - 1; c >= 0; --c) {
    const int64_t t0 = static_cast<int64_t>(c) * kTc;
    const int nv = chunk_len(c);
    float hs[SPL];
#pragma unroll
    for (int j = 0; j < SPL; ++j) hs[j] = hs_next[j];
    stage(c, true, R);
    if (c > 0) {
      fetch(c - 1, true, R);
      fetch_ckpt(c - 1, hs_next);
    }
    // (a) states of the chunk, forward from its checkpoint; partial readout.
    // All kTc tokens, unrolled (past nv: no change, C = 0).
#pragma unroll
    for (int j = 0; j < SPL; ++j) h[j] = hs[j];
#pragma unroll
    for (int t = 0; t < kTc; ++t) {
      const float dt = S.dt[t][lane], du = dt * S.u[t][lane];
      float yp = 0.f;
#pragma unroll
      for (int j = 0; j < SPL; ++j) {
        const int n = warp * SPL + j;
        h[j] = fmaf(ex2_fast(dt * Al[j]), h[j], du * S.Bv[t][n]);
        S.H[t][n][lane] = h[j];
        yp = fmaf(S.Cv[t][n], h[j], yp);
      }
      atomicAdd(&S.part[0][t][lane], yp);
    }
    __syncthreads();
    // (b) the gate's gradient dz = dy · (C·h + D u) · silu'(z); the sums are
    // then cleared for the reverse walk's dΔ
    for (int t = pt; t < kTc; t += NW) {
      if (z && t < nv && ch_ok && SAMBA_CHECK(t0 + t < L && b < (int64_t)gridDim.y)) {
        const float ypre = S.part[0][t][pc] + dsk * S.u[t][pc];
        stv<XT>(p.dz, (b * L + t0 + t) * D + ch_p, ypre * S.dydsz[t][pc]);
      }
      S.part[0][t][pc] = 0.f;
    }
    __syncthreads();
    // (c) the adjoint recurrence, last token first, in groups of G4 tokens
    // whose 2·SPL channel sums each are reduced together.  Tokens past nv
    // (a partial last chunk) contribute nothing and leave g unchanged.
#pragma unroll
    for (int tg = kTc / G4 - 1; tg >= 0; --tg) {
      float q[NV];
#pragma unroll
      for (int i = 0; i < G4; ++i) {
        const int t = tg * G4 + (G4 - 1 - i);
        const bool valid = t < nv;
        const float gyv = valid ? S.gy[t][lane] : 0.f;
        const float dt = valid ? S.dt[t][lane] : 0.f;
        const float uv = valid ? S.u[t][lane] : 0.f;
        const float du = dt * uv;  // rounded as in (a)
        float gB = 0.f, ddt = 0.f;
#pragma unroll
        for (int j = 0; j < SPL; ++j) {
          const int n = warp * SPL + j;
          const float ht = valid ? S.H[t][n][lane] : 0.f;
          const float bv = S.Bv[t][n];
          // exp(Δ A) h_{t-1} = h_t - Δ u B: (a) formed h_t as that sum, so
          // the decayed previous state needs neither h_{t-1} nor the product
          const float dh = ht - du * bv;
          g[j] = fmaf(S.Cv[t][n], gyv, g[j]);
          const float decay = ex2_fast(dt * Al[j]);
          const float gdh = g[j] * dh;
          q[i * 2 * SPL + j] = gyv * ht;       // dC contribution
          q[i * 2 * SPL + SPL + j] = g[j] * du;  // dB contribution
          gB = fmaf(g[j], bv, gB);
          ddt = fmaf(gdh, Al[j] * (1.0f / kLog2e), ddt);
          dAacc[j] = fmaf(gdh, dt, dAacc[j]);
          g[j] *= decay;
        }
        if (valid) {
          atomicAdd(&S.part[0][t][lane], fmaf(uv, gB, ddt));
          atomicAdd(&S.part[1][t][lane], dt * gB);
        }
      }
      int which = 0;
      const float sum = warp_sum_many<NV>(q, lane, &which);
      if ((lane & ((32 / NV) - 1)) == 0) {
        const int i = which / (2 * SPL), k = which % (2 * SPL);
        const int t = tg * G4 + (G4 - 1 - i);
        if (t < nv) S.dbc[k < SPL ? 1 : 0][t][warp * SPL + (k % SPL)] = sum;
      }
    }
    __syncthreads();
    // this block's partial dB, dC rows of the chunk: [t0, t0 + nv) × N, contiguous
    {
      const int64_t BLN = static_cast<int64_t>(gridDim.y) * L * N;
      float* dst = p.part + static_cast<int64_t>(blockIdx.x) * 2 * BLN + (b * L + t0) * N;
      for (int i = tid; i < 2 * nv * N; i += kThreads) {
        const int w = i / (nv * N), r = i - w * (nv * N);
        if (SAMBA_CHECK((b * L + t0) * N + r < BLN)) dst[w * BLN + r] = S.dbc[w][r / N][r % N];
      }
    }
    // (d) du, dΔ, the conv's SiLU; accumulate dD and the conv parameter sums
    for (int t = pt; t < kTc; t += NW) {
      float dcv = 0.f;
      if (t < nv) {
        const float du = dsk * S.gy[t][pc] + S.part[1][t][pc];
        const float ddt = S.part[0][t][pc];
        const int64_t e = (b * L + t0 + t) * D + ch_p;
        if (ch_ok && SAMBA_CHECK(e < (int64_t)gridDim.y * L * D)) p.ddelta[e] = ddt * S.sg[t][pc];
        accD = fmaf(S.gy[t][pc], S.u[t][pc], accD);
        if (fuse) {
          // the conv output before its SiLU, again from the staged inputs
          float pre = cb;
          #pragma unroll
          for (int k = 0; k < 4; ++k)
            if (k < K) pre = fmaf(cw[k], S.x[t + kHalo - (K - 1) + k][pc], pre);
          if (csilu) {
            const float sgp = sigmoid_dev(pre);
            dcv = du * sgp * (1.f + pre * (1.f - sgp));
          } else {
            dcv = du;
          }
          accB += dcv;
          #pragma unroll
          for (int k = 0; k < 4; ++k)
            if (k < K) accW[k] = fmaf(dcv, S.x[t + kHalo - (K - 1) + k][pc], accW[k]);
        } else if (ch_ok) {
          stv<XT>(p.dx, e, du);
        }
      }
      S.dc[t][pc] = dcv;  // rows past nv stay zero: tokens beyond L
    }
    __syncthreads();
    // (e) the conv's input gradient: dx_t = Σ_k w_k dc_{t + K-1-k}
    if (fuse) {
      for (int t = pt; t < nv; t += NW) {
        float v = 0.f;
        #pragma unroll
        for (int k = 0; k < 4; ++k)
          if (k < K) v = fmaf(cw[k], S.dc[t + (K - 1) - k][pc], v);
        if (ch_ok && SAMBA_CHECK(t0 + t < L && b < (int64_t)gridDim.y)) stv<XT>(p.dx, (b * L + t0 + t) * D + ch_p, v);
      }
    }
    __syncthreads();
    // the first rows of this chunk become the halo of the chunk before it
    for (int r = pt; r < kHalo; r += NW) S.dc[kTc + r][pc] = S.dc[r][pc];
    __syncthreads();
  }

  // ------------------------------------------------ epilogue
  if (lane_ok) {
#pragma unroll
    for (int j = 0; j < SPL; ++j) {
      const int n = warp * SPL + j;
      if (p.dh0) p.dh0[(b * D + ch_l) * N + n] = g[j];
      atomicAdd(p.dA + ch_l * N + n, dAacc[j]);
    }
  }
  // gradient of the conv state: entry j holds the input at token j - (K-1)
  if (fuse && p.dconv_state && pt == 0 && ch_ok) {
    for (int j = 0; j < K - 1; ++j) {
      float v = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (k < K && j - k >= 0) v = fmaf(cw[k], S.dc[kTc + (j - k)][pc], v);
      p.dconv_state[(b * D + ch_p) * (K - 1) + j] = v;
    }
  }
  S.red[0][pt][pc] = accD;
  S.red[1][pt][pc] = accB;
  #pragma unroll
  for (int k = 0; k < 4; ++k) S.red[2 + k][pt][pc] = accW[k];
  __syncthreads();
  if (pt == 0 && ch_ok) {
    auto tot = [&](int i) {
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) acc += S.red[i][w][pc];
      return acc;
    };
    if (p.dD) atomicAdd(p.dD + ch_p, tot(0));
    if (fuse) {
      if (p.dconv_b) atomicAdd(p.dconv_b + ch_p, tot(1));
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (k < K) atomicAdd(p.dconv_w + ch_p * K + k, tot(2 + k));
    }
  }
}

// dB, dC = the sum over channel blocks of their partials (four floats per
// thread; the element count 2·B·L·N is a multiple of 4).
__global__ void __launch_bounds__(256) scan_bwd_reduce_kernel(const float4* __restrict__ part, float4* __restrict__ dB,
                                                             float4* __restrict__ dC, int nblk, int64_t bln4) {
  const int64_t n4 = 2 * bln4;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n4; e += (int64_t)gridDim.x * blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k = 0; k < nblk; ++k) {
      const float4 v = part[k * n4 + e];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    if (e < bln4) dB[e] = acc;
    else dC[e - bln4] = acc;
  }
}

template <int N, typename XT, typename YT>
int scan_bwd_go(const ScanBwdParams& p, int64_t B, cudaStream_t s) {
  const size_t smem = sizeof(ScanBwdSmem<N>);
  auto kern = scan_bwd_kernel<N, XT, YT>;
  static PerDeviceOnce attr;
  const int rc = once_per_device(attr, [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) == cudaSuccess
               ? SAMBA_OK
               : fail(SAMBA_ERR_CUDA, "samba_selective_scan_bwd: cannot set shared memory size");
  });
  if (rc != SAMBA_OK) return rc;
  const dim3 grid((unsigned)((p.D + kCh - 1) / kCh), (unsigned)B);
  kern<<<grid, ChunkRegs<N>::kThreads, smem, s>>>(p);
  const int rc2 = check_launch("samba_selective_scan_bwd");
  if (rc2 != SAMBA_OK) return rc2;
  const int64_t bln4 = B * p.L * N / 4;
  const int64_t blocks = std::min<int64_t>((2 * bln4 + 255) / 256, int64_t(sm_count()) * 8);
  scan_bwd_reduce_kernel<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<const float4*>(p.part),
                                                          reinterpret_cast<float4*>(p.dB),
                                                          reinterpret_cast<float4*>(p.dC), (int)grid.x, bln4);
  return check_launch("samba_selective_scan_bwd (reduction)");
}

template <int N>
int scan_bwd_n(const ScanBwdParams& p, int64_t B, int xdt, int ydt, cudaStream_t s) {
  const bool xb = xdt == SAMBA_BF16, yb = ydt == SAMBA_BF16;
  if (xb && yb) return scan_bwd_go<N, __nv_bfloat16, __nv_bfloat16>(p, B, s);
  if (xb) return scan_bwd_go<N, __nv_bfloat16, float>(p, B, s);
  if (yb) return scan_bwd_go<N, float, __nv_bfloat16>(p, B, s);
  return scan_bwd_go<N, float, float>(p, B, s);
}

}  // namespace

// Workspace: the chunk checkpoints [B, ceil(L/16), N, D] fp32, then (at a
// 256-byte boundary) the per-block partials [ceil(D/32)][2][B, L, N] fp32.
static size_t ckpt_bytes(int64_t B, int64_t L, int64_t D, int N) {
  const int64_t nch = (L + kTc - 1) / kTc;
  size_t r = 0;
  if (__builtin_mul_overflow(static_cast<size_t>(B), static_cast<size_t>(nch), &r) ||
      __builtin_mul_overflow(r, static_cast<size_t>(N), &r) || __builtin_mul_overflow(r, static_cast<size_t>(D), &r) ||
      __builtin_mul_overflow(r, sizeof(float), &r) || __builtin_add_overflow(r, size_t(255), &r))
    return SIZE_MAX;
  return r & ~size_t(255);
}

size_t scan_bwd_workspace(int64_t B, int64_t L, int64_t D, int N) {
  const size_t ck = ckpt_bytes(B, L, D, N);
  const int64_t nblk = (D + kCh - 1) / kCh;
  size_t r = 0;
  if (ck == SIZE_MAX || __builtin_mul_overflow(static_cast<size_t>(nblk) * 2, static_cast<size_t>(B), &r) ||
      __builtin_mul_overflow(r, static_cast<size_t>(L), &r) || __builtin_mul_overflow(r, static_cast<size_t>(N), &r) ||
      __builtin_mul_overflow(r, sizeof(float), &r) || __builtin_add_overflow(r, ck, &r))
    return SIZE_MAX;
  return r;
}

int launch_scan_bwd(const samba_scan_bwd_args& a, cudaStream_t s) {
  ScanBwdParams p;
  p.x = a.x;
  p.delta = a.delta;
  p.A = a.A;
  p.Bm = a.Bm;
  p.Cm = a.Cm;
  p.Dskip = a.Dskip;
  p.z = a.z;
  p.conv_w = a.conv_w;
  p.conv_b = a.conv_b;
  p.h0 = a.h0;
  p.conv_state_in = a.conv_state_in;
  p.dy = a.dy;
  p.dx = a.dx;
  p.ddelta = a.ddelta;
  p.dz = a.dz;
  p.dA = a.dA;
  p.dB = a.dB;
  p.dC = a.dC;
  p.dD = a.dD;
  p.dconv_w = a.dconv_w;
  p.dconv_b = a.dconv_b;
  p.dh0 = a.dh0;
  p.dconv_state = a.dconv_state;
  p.ckpt = a.ckpt ? const_cast<float*>(a.ckpt) : reinterpret_cast<float*>(a.workspace);
  p.ckpt_given = a.ckpt != nullptr;
  p.part = reinterpret_cast<float*>(static_cast<unsigned char*>(a.workspace) +
                                    ckpt_bytes(a.batch, a.seqlen, a.dim, a.dstate));
  p.L = a.seqlen;
  p.D = a.dim;
  p.K = a.dconv;
  p.nchunks = static_cast<int>((a.seqlen + kTc - 1) / kTc);
  p.flags = a.flags;
  const int64_t N = a.dstate;
  // the sums the kernel accumulates start from zero
  struct Zero { void* ptr; size_t bytes; };
  const Zero zs[] = {{a.dA, sizeof(float) * a.dim * N},
                     {a.dD, a.dD ? sizeof(float) * a.dim : 0},
                     {a.dconv_w, (a.flags & SAMBA_SCAN_FUSE_CONV) ? sizeof(float) * a.dim * a.dconv : 0},
                     {a.dconv_b, (a.flags & SAMBA_SCAN_FUSE_CONV) && a.dconv_b ? sizeof(float) * a.dim : 0}};
  for (const Zero& zr : zs)
    if (zr.ptr && zr.bytes && cudaMemsetAsync(zr.ptr, 0, zr.bytes, s) != cudaSuccess)
      return fail(SAMBA_ERR_CUDA, "samba_selective_scan_bwd: cannot clear an accumulated output");
  switch (a.dstate) {
    case 4: return scan_bwd_n<4>(p, a.batch, a.x_dtype, a.y_dtype, s);
    case 8: return scan_bwd_n<8>(p, a.batch, a.x_dtype, a.y_dtype, s);
    default: return scan_bwd_n<16>(p, a.batch, a.x_dtype, a.y_dtype, s);
  }
}

}  // namespace samba
