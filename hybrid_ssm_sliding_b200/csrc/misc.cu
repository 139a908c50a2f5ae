// Standalone conv1d and the single-token decode kernels (mamba_step and
// swa_step of the decode loop in the "推理效率" section of the page
// "SAMBA混合注意力状态空间模型"), plus the prefill -> decode ring hand-off.
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "host.hpp"

namespace samba {

int take_status_misc(cudaStream_t s) { return take_status_word(s); }

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float silu_dev(float v) { return __fdividef(v, 1.0f + __expf(-v)); }
__device__ __forceinline__ float softplus_dev(float w) {
  return w > 20.0f ? w : (w > 0.0f ? w + log1pf(__expf(-w)) : log1pf(__expf(w)));
}

template <typename T>
__device__ __forceinline__ float ld_any(const void* p, int64_t i) {
  return to_f32<T>(reinterpret_cast<const T*>(p)[i]);
}

// ---------------------------------------------------------------- conv1d
// u[b,t,c] = bias[c] + sum_k w[c,k] x[b,t-K+1+k,c] (earlier inputs from the
// conv state), then SiLU.  One thread per output element.
template <typename XT, typename UT>
__global__ void conv1d_kernel(const XT* __restrict__ x, const float* __restrict__ w, const float* __restrict__ bias,
                              const float* __restrict__ cs_in, UT* __restrict__ u, int64_t B, int64_t L, int64_t D,
                              int K, int silu) {
  const int64_t n = B * L * D;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = e % D;
    const int64_t t = (e / D) % L;
    const int64_t b = e / (D * L);
    float acc = bias ? bias[c] : 0.f;
    for (int k = 0; k < K; ++k) {
      const int64_t tt = t - (K - 1) + k;
      float xv;
      if (tt >= 0) xv = to_f32<XT>(x[(b * L + tt) * D + c]);
      else xv = cs_in ? cs_in[(b * D + c) * (K - 1) + (K - 1) + tt] : 0.f;
      acc = fmaf(w[c * K + k], xv, acc);
    }
    if (silu) acc = silu_dev(acc);
    u[e] = from_f32<UT>(acc);
  }
}

template <typename XT>
__global__ void conv_state_kernel(const XT* __restrict__ x, const float* __restrict__ cs_in,
                                  float* __restrict__ cs_out, int64_t B, int64_t L, int64_t D, int K) {
  const int64_t n = B * D * (K - 1);
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int j = (int)(e % (K - 1));
    const int64_t c = (e / (K - 1)) % D;
    const int64_t b = e / ((K - 1) * D);
    const int64_t src = L + j - (K - 1);
    float v;
    if (src >= 0) v = to_f32<XT>(x[(b * L + src) * D + c]);
    else v = cs_in ? cs_in[(b * D + c) * (K - 1) + (K - 1) + src] : 0.f;
    cs_out[e] = v;
  }
}

// One position (L = 1) with the conv state carried: one thread per (b, c)
// reads the channel's K-1 earlier inputs and x, writes u and the shifted
// state.  A thread reads everything it needs before it writes, and no other
// thread touches that channel's state, so cs_out may be cs_in.
template <typename XT, typename UT>
__global__ void conv1d_step_kernel(const XT* __restrict__ x, const float* __restrict__ w,
                                   const float* __restrict__ bias, const float* cs_in, UT* __restrict__ u,
                                   float* cs_out, int64_t B, int64_t D, int K, int silu) {
  const int64_t n = B * D;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = e % D;
    float xp[4];
    for (int k = 0; k < K - 1; ++k) xp[k] = cs_in ? cs_in[e * (K - 1) + k] : 0.f;
    xp[K - 1] = to_f32<XT>(x[e]);
    float acc = bias ? bias[c] : 0.f;
    for (int k = 0; k < K; ++k) acc = fmaf(w[c * K + k], xp[k], acc);
    if (silu) acc = silu_dev(acc);
    u[e] = from_f32<UT>(acc);
    for (int k = 0; k < K - 1; ++k) cs_out[e * (K - 1) + k] = xp[k + 1];
  }
}

template <typename XT, typename UT>
static void conv1d_go(const void* x, const float* w, const float* bias, const float* cs_in, void* u, float* cs_out,
                      int64_t B, int64_t L, int64_t D, int K, int silu, cudaStream_t s) {
  const int64_t n = B * L * D;
  const int threads = 256;
  const int blocks = (int)std::min<int64_t>((n + threads - 1) / threads, (int64_t)sm_count() * 16);
  if (L == 1 && cs_out) {
    conv1d_step_kernel<XT, UT><<<blocks, threads, 0, s>>>(reinterpret_cast<const XT*>(x), w, bias, cs_in,
                                                           reinterpret_cast<UT*>(u), cs_out, B, D, K, silu);
    return;
  }
  conv1d_kernel<XT, UT><<<blocks, threads, 0, s>>>(reinterpret_cast<const XT*>(x), w, bias, cs_in,
                                                    reinterpret_cast<UT*>(u), B, L, D, K, silu);
  if (cs_out) {
    const int64_t m = B * D * (K - 1);
    conv_state_kernel<XT><<<(int)std::min<int64_t>((m + 255) / 256, 4096), 256, 0, s>>>(
        reinterpret_cast<const XT*>(x), cs_in, cs_out, B, L, D, K);
  }
}

int launch_conv1d(const void* x, int x_dtype, const float* w, const float* bias, const float* cs_in, void* u,
                  int u_dtype, float* cs_out, int64_t B, int64_t L, int64_t D, int K, int silu, cudaStream_t s) {
  const bool xb = x_dtype == SAMBA_BF16, ub = u_dtype == SAMBA_BF16;
  if (xb && ub) conv1d_go<__nv_bfloat16, __nv_bfloat16>(x, w, bias, cs_in, u, cs_out, B, L, D, K, silu, s);
  else if (xb) conv1d_go<__nv_bfloat16, float>(x, w, bias, cs_in, u, cs_out, B, L, D, K, silu, s);
  else if (ub) conv1d_go<float, __nv_bfloat16>(x, w, bias, cs_in, u, cs_out, B, L, D, K, silu, s);
  else conv1d_go<float, float>(x, w, bias, cs_in, u, cs_out, B, L, D, K, silu, s);
  return check_launch("samba_conv1d_fwd");
}

// -------------------------------------------------------------- scan step
// Four threads per (batch, channel), each holding N/4 of its states (one
// channel per aligned group of four lanes); the C·h partials meet through two
// shuffles.  Same arithmetic as the prefill kernel with L = 1.  Every load
// that does not depend on another is issued first (state, A, B, C as vectors;
// conv taps and state for K <= 4 in registers), so that one round trip to
// memory covers them all.
template <int NS>
__device__ __forceinline__ void ld_states(float (&v)[NS], const float* p) {
  if constexpr (NS == 4) {
    const float4 t = *reinterpret_cast<const float4*>(p);
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
  } else if constexpr (NS == 2) {
    const float2 t = *reinterpret_cast<const float2*>(p);
    v[0] = t.x; v[1] = t.y;
  } else {
#pragma unroll
    for (int n = 0; n < NS; ++n) v[n] = p[n];
  }
}
template <int NS>
__device__ __forceinline__ void st_states(float* p, const float (&v)[NS]) {
  if constexpr (NS == 4) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  } else if constexpr (NS == 2) {
    *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
  } else {
#pragma unroll
    for (int n = 0; n < NS; ++n) p[n] = v[n];
  }
}

template <int N, typename XT, typename YT>
__global__ void __launch_bounds__(256) scan_step_kernel(
    float* __restrict__ h, float* __restrict__ cs, const XT* __restrict__ x_t, const XT* __restrict__ z_t,
    const float* __restrict__ delta_t, const float* __restrict__ B_t, const float* __restrict__ C_t,
    const float* __restrict__ A, const float* __restrict__ Dskip, const float* __restrict__ conv_w,
    const float* __restrict__ conv_b, YT* __restrict__ y_t, int64_t D, int K, uint32_t flags) {
  constexpr int TPC = 4, NS = N / TPC;
  const int64_t b = blockIdx.y;
  const int64_t c = (int64_t)blockIdx.x * (blockDim.x / TPC) + threadIdx.x / TPC;
  const int j = threadIdx.x % TPC;
  if (c >= D) return;  // whole groups of four leave together
  const unsigned gmask = 0xFu << (threadIdx.x & 28);
  const int64_t e = b * D + c;
  const bool fuse = (flags & SAMBA_SCAN_FUSE_CONV) != 0;
  // ---- loads
  const float xv = to_f32<XT>(x_t[e]);
  const float wr = delta_t[e];
  float hv[NS], av[NS], bv[NS], cv[NS];
  float* hp = h + e * N + j * NS;
  ld_states<NS>(hv, hp);
  ld_states<NS>(av, A + c * N + j * NS);
  ld_states<NS>(bv, B_t + b * N + j * NS);
  ld_states<NS>(cv, C_t + b * N + j * NS);
  float* st = cs + e * (K - 1);
  float sv[3] = {0.f, 0.f, 0.f}, cw[3] = {0.f, 0.f, 0.f}, wlast = 0.f, cbias = 0.f;
  if (fuse) {
#pragma unroll
    for (int k = 0; k < 3; ++k)
      if (k < K - 1) {
        sv[k] = st[k];
        cw[k] = conv_w[c * K + k];
      }
    wlast = conv_w[c * K + K - 1];
    if (conv_b) cbias = conv_b[c];
  }
  const float zv = (z_t && j == 0) ? to_f32<XT>(z_t[e]) : 0.f;
  const float dsk = (Dskip && j == 0) ? Dskip[c] : 0.f;
  // ---- conv and the state shift
  float u;
  if (fuse) {
    float acc = cbias;
#pragma unroll
    for (int k = 0; k < 3; ++k)
      if (k < K - 1) acc = fmaf(cw[k], sv[k], acc);
    acc = fmaf(wlast, xv, acc);
    __syncwarp(gmask);  // every thread of the group has read the old state
    if (j == 0) {
#pragma unroll
      for (int k = 0; k < 2; ++k)
        if (k + 1 < K - 1) st[k] = sv[k + 1];
      st[K - 2] = xv;
    }
    u = (flags & SAMBA_SCAN_CONV_SILU) ? silu_dev(acc) : acc;
  } else {
    u = xv;
  }
  const float dlt = (flags & SAMBA_SCAN_DELTA_SOFTPLUS) ? softplus_dev(wr) : wr;
  const float du = dlt * u;
  constexpr float kLog2e = 1.4426950408889634f;
  float acc = 0.f;
#pragma unroll
  for (int n = 0; n < NS; ++n) {
    hv[n] = fmaf(ex2_approx(dlt * (av[n] * kLog2e)), hv[n], du * bv[n]);
    acc = fmaf(cv[n], hv[n], acc);
  }
  st_states<NS>(hp, hv);
  acc += __shfl_xor_sync(gmask, acc, 1);
  acc += __shfl_xor_sync(gmask, acc, 2);
  if (j == 0) {
    float yv = acc + (Dskip ? dsk * u : 0.f);
    if (z_t) yv *= silu_dev(zv);
    y_t[e] = from_f32<YT>(yv);
  }
}

template <int N, typename XT, typename YT>
static void scan_step_go(float* h, float* cs, const void* x_t, const void* z_t, const float* delta_t, const float* B_t,
                         const float* C_t, const float* A, const float* Dskip, const float* conv_w,
                         const float* conv_b, void* y_t, int64_t B, int64_t D, int K, uint32_t flags,
                         cudaStream_t s) {
  const dim3 grid((unsigned)((D + 63) / 64), (unsigned)B);
  scan_step_kernel<N, XT, YT><<<grid, 256, 0, s>>>(
      h, cs, reinterpret_cast<const XT*>(x_t), reinterpret_cast<const XT*>(z_t), delta_t, B_t, C_t, A, Dskip, conv_w,
      conv_b, reinterpret_cast<YT*>(y_t), D, K, flags);
}

template <int N>
static void scan_step_n(float* h, float* cs, const void* x_t, int xdt, const void* z_t, const float* delta_t,
                        const float* B_t, const float* C_t, const float* A, const float* Dskip, const float* conv_w,
                        const float* conv_b, void* y_t, int ydt, int64_t B, int64_t D, int K, uint32_t flags,
                        cudaStream_t s) {
  const bool xb = xdt == SAMBA_BF16, yb = ydt == SAMBA_BF16;
  if (xb && yb) scan_step_go<N, __nv_bfloat16, __nv_bfloat16>(h, cs, x_t, z_t, delta_t, B_t, C_t, A, Dskip, conv_w, conv_b, y_t, B, D, K, flags, s);
  else if (xb) scan_step_go<N, __nv_bfloat16, float>(h, cs, x_t, z_t, delta_t, B_t, C_t, A, Dskip, conv_w, conv_b, y_t, B, D, K, flags, s);
  else if (yb) scan_step_go<N, float, __nv_bfloat16>(h, cs, x_t, z_t, delta_t, B_t, C_t, A, Dskip, conv_w, conv_b, y_t, B, D, K, flags, s);
  else scan_step_go<N, float, float>(h, cs, x_t, z_t, delta_t, B_t, C_t, A, Dskip, conv_w, conv_b, y_t, B, D, K, flags, s);
}

int launch_scan_step(float* h, float* conv_state, const void* x_t, int x_dtype, const void* z_t, int z_dtype,
                     const float* delta_t, const float* B_t, const float* C_t, const float* A, const float* Dskip,
                     const float* conv_w, const float* conv_b, void* y_t, int y_dtype, int64_t B, int64_t D, int N,
                     int K, uint32_t flags, cudaStream_t s) {
  if (z_t && z_dtype != x_dtype) return fail(SAMBA_ERR_UNSUPPORTED, "samba_scan_step: z dtype must equal x dtype");
  const void* vec[] = {h, A, B_t, C_t};
  for (const void* p : vec)
    if (!aligned16(p)) return fail(SAMBA_ERR_INVALID_ARG, "samba_scan_step: h, A, B_t, C_t must be 16-byte aligned");
  switch (N) {
    case 4: scan_step_n<4>(h, conv_state, x_t, x_dtype, z_t, delta_t, B_t, C_t, A, Dskip, conv_w, conv_b, y_t, y_dtype, B, D, K, flags, s); break;
    case 8: scan_step_n<8>(h, conv_state, x_t, x_dtype, z_t, delta_t, B_t, C_t, A, Dskip, conv_w, conv_b, y_t, y_dtype, B, D, K, flags, s); break;
    default: scan_step_n<16>(h, conv_state, x_t, x_dtype, z_t, delta_t, B_t, C_t, A, Dskip, conv_w, conv_b, y_t, y_dtype, B, D, K, flags, s); break;
  }
  return check_launch("samba_scan_step");
}

// -------------------------------------------------------------- ring fill
// Copies 16-byte chunks of the last min(L, W) positions into their slots.
__global__ void ring_fill_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v, uint4* __restrict__ kr,
                                 uint4* __restrict__ vr, int64_t* __restrict__ pos, int64_t B, int64_t L, int64_t W,
                                 int row_chunks) {
  const int64_t keep = L < W ? L : W;
  const int64_t n = B * keep * row_chunks;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t ch = e % row_chunks;
    const int64_t r = (e / row_chunks) % keep;
    const int64_t b = e / (row_chunks * keep);
    const int64_t p = L - keep + r;
    const int64_t slot = p % W;
    kr[(b * W + slot) * row_chunks + ch] = k[(b * L + p) * row_chunks + ch];
    vr[(b * W + slot) * row_chunks + ch] = v[(b * L + p) * row_chunks + ch];
  }
  if (blockIdx.x == 0)
    for (int64_t b = threadIdx.x; b < B; b += blockDim.x) pos[b] = L;
}

int launch_ring_fill(const void* k, const void* v, int64_t L, void* k_ring, void* v_ring, int64_t* pos, int64_t B,
                     int Hkv, int d, int64_t W, cudaStream_t s) {
  const int row_chunks = Hkv * d * 2 / 16;
  const int64_t n = B * std::min(L, W) * row_chunks;
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, (int64_t)sm_count() * 8));
  ring_fill_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<const uint4*>(k), reinterpret_cast<const uint4*>(v),
                                          reinterpret_cast<uint4*>(k_ring), reinterpret_cast<uint4*>(v_ring), pos, B,
                                          L, W, row_chunks);
  return check_launch("samba_swa_ring_fill");
}

// --------------------------------------------------------------- SWA step
// Split over the window: CTA (split, kv head g, batch b) handles CH consecutive
// positions of the window for the `group` query heads of g, writing a partial
// (max, sum, unnormalised output) per head; a second kernel combines the
// splits.  The newest position is read from k_t/v_t, which split 0 also
// stores into its ring slot (that slot held a position outside the window, so
// no other CTA reads it in this step).  The CTA loads its chunk's K and V
// rows into shared memory in one burst of 16-byte chunks (all rows in flight
// at once, a warp's load covering whole rows); the scores K·qᵀ (pos x heads) and
// the outputs P·V (heads x head dim) are bf16 tensor-core products
// (mma m16n8k16, fp32 accumulate), P rounded to bf16 as in the prefill.
template <int HD> struct StepCfg {
  static constexpr int CH = HD <= 64 ? 128 : 64;  // positions per CTA (= threads)
  static constexpr int NWARP = CH / 32;
  static constexpr int KP = HD + 8;                // row pitch of K, V, q in bf16 (conflict-free fragments)
  static constexpr int PP = CH + 8;                // row pitch of P in bf16
  // shared memory: V, then K + q during the scores, reused for scores + P
  static constexpr int V_BYTES = CH * KP * 2;
  static constexpr int KQ_BYTES = CH * KP * 2 + 16 * KP * 2;
  static constexpr int SP_BYTES = 16 * CH * 4 + 16 * PP * 2;
  static constexpr int SMEM = V_BYTES + (KQ_BYTES > SP_BYTES ? KQ_BYTES : SP_BYTES);
};

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int HD>
__global__ void __launch_bounds__(StepCfg<HD>::CH) swa_step_split_kernel(
    const __nv_bfloat16* __restrict__ q_t, const __nv_bfloat16* __restrict__ k_t,
    const __nv_bfloat16* __restrict__ v_t, __nv_bfloat16* __restrict__ k_ring, __nv_bfloat16* __restrict__ v_ring,
    const int64_t* __restrict__ pos, float* __restrict__ ws, int Hq, int Hkv, int64_t W, float scale_log2,
    int nsplit) {
  using Cfg = StepCfg<HD>;
  constexpr int CH = Cfg::CH, NWARP = Cfg::NWARP, KP = Cfg::KP, PP = Cfg::PP;
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int group = Hq / Hkv;  // <= 16
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Loads that do not depend on pos go first, so that they are in flight
  // together with the read of pos: the group's query rows (16-byte chunks of
  // the zero-padded 16-row tile) and, in split 0, the new key/value row.
  constexpr int QCH = 16 * HD / 8, QPT = (QCH + CH - 1) / CH, RCH = HD / 8;
  const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);
  uint4 qraw[QPT];
#pragma unroll
  for (int j = 0; j < QPT; ++j) {
    const int i = tid + j * CH, hh = i / RCH, c = i % RCH;
    qraw[j] = (i < QCH && hh < group)
                  ? reinterpret_cast<const uint4*>(q_t + ((int64_t)b * Hq + g * group + hh) * HD)[c]
                  : zero4;
  }
  const int64_t noff = ((int64_t)b * Hkv + g) * HD;
  uint4 knew = zero4, vnew = zero4;
  if (split == 0 && tid < RCH) {
    knew = reinterpret_cast<const uint4*>(k_t + noff)[tid];
    vnew = reinterpret_cast<const uint4*>(v_t + noff)[tid];
  }
  const int64_t p = pos[b];
  const int64_t lo = p - W + 1 > 0 ? p - W + 1 : 0;
  const int64_t a0 = lo + (int64_t)split * CH;
  // positions a0 .. a0 + n_here - 1 of this chunk are valid; their ring slots
  // are consecutive modulo W, starting at slot0 (one 64-bit remainder per CTA)
  const int n_here = (int)(p - a0 + 1 < CH ? (p - a0 + 1 > 0 ? p - a0 + 1 : 0) : CH);
  const int slot0 = (int)(a0 % W);
  const int Wi = (int)W;
  __shared__ __align__(16) unsigned char sm[Cfg::SMEM];
  __nv_bfloat16* Vs = reinterpret_cast<__nv_bfloat16*>(sm);                              // [CH][KP]
  __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(sm + Cfg::V_BYTES);               // [CH][KP]
  __nv_bfloat16* Qs = Ks + CH * KP;                                                       // [16][KP]
  float* Sc = reinterpret_cast<float*>(sm + Cfg::V_BYTES);                                // [16][CH] (after K)
  __nv_bfloat16* Ps = reinterpret_cast<__nv_bfloat16*>(sm + Cfg::V_BYTES + 16 * CH * 4);  // [16][PP]
  __shared__ float red_m[16], red_l[16];

  const int gq = lane >> 2, tq = lane & 3;  // mma fragment coordinates
  // K and V rows of the chunk to shared memory (zeros past the window), as
  // 16-byte chunks: consecutive threads take consecutive chunks of a row, so
  // a warp's load covers whole rows (RCH chunks each); the newest position
  // comes from k_t / v_t.
  {
    uint4 kraw[RCH], vraw[RCH];
#pragma unroll
    for (int i = 0; i < RCH; ++i) {
      const int ig = tid + i * CH, r = ig / RCH, c = ig % RCH;
      const bool valid = r < n_here;
      int slot = slot0 + r;
      slot = slot >= Wi ? slot - Wi : slot;
      const bool is_new = a0 + r == p;
      const int64_t roff = (((int64_t)b * W + (valid ? slot : 0)) * Hkv + g) * HD;
      const uint4* krow = reinterpret_cast<const uint4*>(is_new ? k_t + noff : k_ring + roff);
      const uint4* vrow = reinterpret_cast<const uint4*>(is_new ? v_t + noff : v_ring + roff);
      kraw[i] = valid ? krow[c] : zero4;
      vraw[i] = valid ? vrow[c] : zero4;
    }
#pragma unroll
    for (int i = 0; i < RCH; ++i) {
      const int ig = tid + i * CH, r = ig / RCH, c = ig % RCH;
      reinterpret_cast<uint4*>(Ks + r * KP)[c] = kraw[i];
      reinterpret_cast<uint4*>(Vs + r * KP)[c] = vraw[i];
    }
  }
#pragma unroll
  for (int j = 0; j < QPT; ++j) {
    const int i = tid + j * CH;
    if (i < QCH) reinterpret_cast<uint4*>(Qs + (i / RCH) * KP)[i % RCH] = qraw[j];
  }
  if (split == 0 && tid < RCH) {  // the new key/value into its slot
    const int64_t roff = (((int64_t)b * W + p % W) * Hkv + g) * HD;
    reinterpret_cast<uint4*>(k_ring + roff)[tid] = knew;
    reinterpret_cast<uint4*>(v_ring + roff)[tid] = vnew;
  }
  __syncthreads();

  // scores: warp w takes positions [32w, 32w + 32) (two m16 tiles) against
  // the 16 (zero-padded) head rows (two n8 tiles), k over the head dim
  float sacc[2][2][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[mt][nt][e] = 0.f;
#pragma unroll
  for (int ks = 0; ks < HD / 16; ++ks) {
    const int kc = 16 * ks + 2 * tq;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      const int r0 = 32 * warp + 16 * mt + gq;
      const uint32_t a0r = *reinterpret_cast<const uint32_t*>(Ks + r0 * KP + kc);
      const uint32_t a1r = *reinterpret_cast<const uint32_t*>(Ks + (r0 + 8) * KP + kc);
      const uint32_t a2r = *reinterpret_cast<const uint32_t*>(Ks + r0 * KP + kc + 8);
      const uint32_t a3r = *reinterpret_cast<const uint32_t*>(Ks + (r0 + 8) * KP + kc + 8);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int n = 8 * nt + gq;
        const uint32_t b0r = *reinterpret_cast<const uint32_t*>(Qs + n * KP + kc);
        const uint32_t b1r = *reinterpret_cast<const uint32_t*>(Qs + n * KP + kc + 8);
        mma_bf16_16816(sacc[mt][nt], a0r, a1r, a2r, a3r, b0r, b1r);
      }
    }
  }
  __syncthreads();  // K and q are read: their space now holds the scores and P
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = 32 * warp + 16 * mt + gq + (e >= 2 ? 8 : 0);  // position
        const int col = 8 * nt + 2 * tq + (e & 1);                      // head
        Sc[col * CH + row] = row < n_here ? sacc[mt][nt][e] * scale_log2 : -INFINITY;
      }
  __syncthreads();
  // per head max and exp-sum (one warp per head, heads strided over the
  // warps); P in bf16, rows past the group zero
  for (int hh = warp; hh < 16; hh += NWARP) {
    if (hh >= group) {
      for (int i = lane; i < CH; i += 32) Ps[hh * PP + i] = __float2bfloat16_rn(0.f);
      continue;
    }
    float m = -INFINITY;
    for (int i = lane; i < CH; i += 32) m = fmaxf(m, Sc[hh * CH + i]);
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float mu = (m == -INFINITY) ? 0.f : m;
    float l = 0.f;
    for (int i = lane; i < CH; i += 32) {
      const __nv_bfloat16 e = __float2bfloat16_rn(ex2_approx(Sc[hh * CH + i] - mu));
      Ps[hh * PP + i] = e;
      l += __bfloat162float(e);  // the sum of the probabilities P·V uses
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      red_m[hh] = m;
      red_l[hh] = l;
    }
  }
  __syncthreads();
  // outputs: heads (m16) x head dim (n8 tiles over the warps), k over positions
  for (int nt = warp; nt < HD / 8; nt += NWARP) {
    float oacc[4] = {0.f, 0.f, 0.f, 0.f};
    const int n = 8 * nt + gq;  // head-dim column of the B fragment
#pragma unroll
    for (int ks = 0; ks < CH / 16; ++ks) {
      const int kc = 16 * ks + 2 * tq;
      const uint32_t a0r = *reinterpret_cast<const uint32_t*>(Ps + gq * PP + kc);
      const uint32_t a1r = *reinterpret_cast<const uint32_t*>(Ps + (gq + 8) * PP + kc);
      const uint32_t a2r = *reinterpret_cast<const uint32_t*>(Ps + gq * PP + kc + 8);
      const uint32_t a3r = *reinterpret_cast<const uint32_t*>(Ps + (gq + 8) * PP + kc + 8);
      const unsigned short* vb = reinterpret_cast<const unsigned short*>(Vs);
      const uint32_t b0r = (uint32_t)vb[kc * KP + n] | ((uint32_t)vb[(kc + 1) * KP + n] << 16);
      const uint32_t b1r = (uint32_t)vb[(kc + 8) * KP + n] | ((uint32_t)vb[(kc + 9) * KP + n] << 16);
      mma_bf16_16816(oacc, a0r, a1r, a2r, a3r, b0r, b1r);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int hh = gq + (e >= 2 ? 8 : 0);
      const int dd = 8 * nt + 2 * tq + (e & 1);
      if (hh < group) {
        float* dst = ws + ((((int64_t)b * Hq + g * group + hh) * nsplit + split) * (HD + 2));
        dst[2 + dd] = oacc[e];
        if (dd == 0) {
          dst[0] = red_m[hh];
          dst[1] = red_l[hh];
        }
      }
    }
  }
}

template <int HD>
__global__ void swa_step_combine_kernel(const float* __restrict__ ws, __nv_bfloat16* __restrict__ o_t,
                                        int64_t* __restrict__ pos, int Hq, int nsplit) {
  const int hq = blockIdx.x, b = blockIdx.y;
  const int dd = threadIdx.x;
  const float* base = ws + ((int64_t)b * Hq + hq) * nsplit * (HD + 2);
  // the loops are unrolled so that the loads of several splits are in flight
  float M = -INFINITY;
#pragma unroll 8
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, base[s * (HD + 2)]);
  float l = 0.f, acc = 0.f;
#pragma unroll 8
  for (int s = 0; s < nsplit; ++s) {
    const float m = base[s * (HD + 2)];
    const float f = (m == -INFINITY) ? 0.f : ex2_approx(m - M);
    l = fmaf(base[s * (HD + 2) + 1], f, l);
    acc = fmaf(base[s * (HD + 2) + 2 + dd], f, acc);
  }
  o_t[((int64_t)b * Hq + hq) * HD + dd] = __float2bfloat16_rn(acc / l);
  if (hq == 0 && dd == 0) pos[b] += 1;
}

// Bytes of split partials: (max, sum, d outputs) per (batch, query head,
// split).  SIZE_MAX when the product does not fit in size_t, so that no
// workspace (and no built-in scratch) is ever taken as large enough.
size_t swa_step_workspace(int64_t B, int Hq, int d, int64_t W) {
  const int ch = d <= 64 ? StepCfg<64>::CH : StepCfg<128>::CH;
  const uint64_t nsplit = static_cast<uint64_t>((W + ch - 1) / ch);
  uint64_t n = 0;
  if (__builtin_mul_overflow(static_cast<uint64_t>(B), static_cast<uint64_t>(Hq), &n) ||
      __builtin_mul_overflow(n, nsplit, &n) || __builtin_mul_overflow(n, static_cast<uint64_t>(d + 2), &n) ||
      __builtin_mul_overflow(n, static_cast<uint64_t>(sizeof(float)), &n) || n > SIZE_MAX)
    return SIZE_MAX;
  return static_cast<size_t>(n);
}

template <int HD>
static void swa_step_go(const void* q_t, const void* k_t, const void* v_t, void* k_ring, void* v_ring, int64_t* pos,
                        void* o_t, int64_t B, int Hq, int Hkv, int64_t W, float scale, void* ws, cudaStream_t s) {
  constexpr int CH = StepCfg<HD>::CH;
  const int nsplit = (int)((W + CH - 1) / CH);
  dim3 g1(nsplit, Hkv, (unsigned)B);
  swa_step_split_kernel<HD><<<g1, CH, 0, s>>>(
      reinterpret_cast<const __nv_bfloat16*>(q_t), reinterpret_cast<const __nv_bfloat16*>(k_t),
      reinterpret_cast<const __nv_bfloat16*>(v_t), reinterpret_cast<__nv_bfloat16*>(k_ring),
      reinterpret_cast<__nv_bfloat16*>(v_ring), pos, reinterpret_cast<float*>(ws), Hq, Hkv, W,
      scale * 1.4426950408889634f, nsplit);
  dim3 g2(Hq, (unsigned)B);
  swa_step_combine_kernel<HD><<<g2, HD, 0, s>>>(reinterpret_cast<const float*>(ws),
                                                 reinterpret_cast<__nv_bfloat16*>(o_t), pos, Hq, nsplit);
}

int launch_swa_step(const void* q_t, const void* k_t, const void* v_t, void* k_ring, void* v_ring, int64_t* pos,
                    void* o_t, int64_t B, int Hq, int Hkv, int d, int64_t W, float scale, void* ws, cudaStream_t s) {
  if (B > 65535) return fail(SAMBA_ERR_UNSUPPORTED, "samba_swa_step: batch too large");
  switch (d) {
    case 16: swa_step_go<16>(q_t, k_t, v_t, k_ring, v_ring, pos, o_t, B, Hq, Hkv, W, scale, ws, s); break;
    case 32: swa_step_go<32>(q_t, k_t, v_t, k_ring, v_ring, pos, o_t, B, Hq, Hkv, W, scale, ws, s); break;
    case 64: swa_step_go<64>(q_t, k_t, v_t, k_ring, v_ring, pos, o_t, B, Hq, Hkv, W, scale, ws, s); break;
    default: swa_step_go<128>(q_t, k_t, v_t, k_ring, v_ring, pos, o_t, B, Hq, Hkv, W, scale, ws, s); break;
  }
  return check_launch("samba_swa_step");
}

}  // namespace samba

// ------------------------------------------------------- bounded-wait self-test
namespace samba {

// One thread waits on a barrier that expects one arrival which never comes.
__global__ void selftest_wait_kernel() {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
    (void)mbar_wait(&bar, 0, &abort_flag);  // gives up after the limit, records the timeout
  }
}

int launch_selftest_wait(cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>();
  return check_launch("samba_selftest_wait_timeout");
}

}  // namespace samba

// ------------------------------------------- SWA step without allocations
// Scratch for samba_swa_step_noalloc: the split partials of swa_step live in
// this file-scope device array instead of caller-provided workspace.  Every
// GPU that loads the library holds it (4 MiB) until the process exits.

namespace samba {

constexpr size_t kSwaStepScratchBytes = size_t(4) << 20;
static __device__ __align__(256) unsigned char g_swa_step_scratch[kSwaStepScratchBytes];

// In host code g_swa_step_scratch names a host-side stand-in, not device
// memory: its device address is looked up with cudaGetSymbolAddress, with
// the calling device current, and passed to the kernels.  The lookup runs on
// every call (it is a table lookup once the module is loaded), so that the
// address stays right after cudaDeviceReset, which reloads the module and
// may place the array elsewhere.
static int scratch_address(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_swa_step_scratch);
  if (e != cudaSuccess || !p)
    return fail(SAMBA_ERR_CUDA, "samba_swa_step_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
  *out = p;
  return SAMBA_OK;
}

int launch_swa_step_noalloc(const void* q_t, const void* k_t, const void* v_t, void* k_ring, void* v_ring,
                            int64_t* pos, void* o_t, int64_t B, int Hq, int Hkv, int d, int64_t W, float scale,
                            cudaStream_t s) {
  const size_t need = swa_step_workspace(B, Hq, d, W);
  if (need > kSwaStepScratchBytes)
    return fail(SAMBA_ERR_WORKSPACE,
                "samba_swa_step_noalloc: these sizes need %zu bytes of scratch but the built-in array holds %zu; "
                "call samba_swa_step with a workspace instead",
                need, kSwaStepScratchBytes);
  void* ws = nullptr;
  const int rc = scratch_address(&ws);
  if (rc != SAMBA_OK) return rc;
  return launch_swa_step(q_t, k_t, v_t, k_ring, v_ring, pos, o_t, B, Hq, Hkv, d, W, scale, ws, s);
}

}  // namespace samba
