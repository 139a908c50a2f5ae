// Standalone conv1d and the single-token decode kernels (mamba_step and
// swa_step of the decode loop in the "推理效率" section of the page
// "SAMBA混合注意力状态空间模型"), plus the prefill -> decode ring hand-off.
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "host.hpp"
#include "pdl.cuh"

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
  pdl_launch_dependents();
  pdl_wait();
  const int64_t n = B * D;
  // The window [state (K - 1 values), x] sits at the end of four registers:
  // v[j] holds tap k = j - (4 - K), so every index is fixed once the loops
  // are unrolled (K is 2..4) and the taps never go to local memory.
  const int off = 4 - K;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = e % D;
    float v[4];
#pragma unroll
    for (int j = 0; j < 3; ++j) v[j] = (j >= off && cs_in) ? cs_in[e * (K - 1) + (j - off)] : 0.f;
    v[3] = to_f32<XT>(x[e]);
    float acc = bias ? bias[c] : 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (j >= off) acc = fmaf(w[c * K + (j - off)], v[j], acc);
    if (silu) acc = silu_dev(acc);
    if (!SAMBA_CHECK(e >= 0 && e < n && K <= 4)) continue;
    u[e] = from_f32<UT>(acc);
#pragma unroll
    for (int j = 1; j < 4; ++j)
      if (j > off) cs_out[e * (K - 1) + (j - off - 1)] = v[j];
  }
}

template <typename XT, typename UT>
static void conv1d_go(const void* x, const float* w, const float* bias, const float* cs_in, void* u, float* cs_out,
                      int64_t B, int64_t L, int64_t D, int K, int silu, cudaStream_t s) {
  const int64_t n = B * L * D;
  const int threads = 256;
  const int blocks = (int)std::min<int64_t>((n + threads - 1) / threads, (int64_t)sm_count() * 16);
  if (L == 1 && cs_out) {  // a decode step: launched as a programmatic dependent (pdl.cuh)
    launch_pdl(conv1d_step_kernel<XT, UT>, dim3(blocks), dim3(threads), 0, s, reinterpret_cast<const XT*>(x), w,
               bias, cs_in, reinterpret_cast<UT*>(u), cs_out, B, D, K, silu);
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
  pdl_launch_dependents();
  pdl_wait();  // every input and the state come from earlier kernels
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
  if (SAMBA_CHECK(b < (int64_t)gridDim.y && c < D)) st_states<NS>(hp, hv);
  acc += __shfl_xor_sync(gmask, acc, 1);
  acc += __shfl_xor_sync(gmask, acc, 2);
  if (j == 0 && SAMBA_CHECK(e < (int64_t)gridDim.y * D)) {
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
  launch_pdl(scan_step_kernel<N, XT, YT>, grid, dim3(256), 0, s, h, cs, reinterpret_cast<const XT*>(x_t),
             reinterpret_cast<const XT*>(z_t), delta_t, B_t, C_t, A, Dskip, conv_w, conv_b,
             reinterpret_cast<YT*>(y_t), D, K, flags);
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
// Split over the ring: CTA (split, kv head g, batch b) takes the ring slots
// [split * chunk, min(W, (split + 1) * chunk)) for the `group` query heads of
// g and writes one partial (max, sum, unnormalised output) per head; a second
// kernel, launched as its programmatic dependent, combines the splits and
// advances pos once every split CTA has read it.  Softmax does not depend on
// the order of the keys, so a CTA works on slots, not positions: slot j holds
// a position of the window exactly when j <= p (p = pos[b], the position of
// the new token; for p >= W every slot does), and the new key and value (slot
// p mod W) come from k_t / v_t, which the CTA owning that slot also stores
// into the ring (no CTA of this step reads that slot from the ring).
//
// K and V stream through shared memory in sub-chunks of 64 slots, one tensor
// TMA copy per matrix (and 64-wide column panel), STG - 1 sub-chunks in
// flight.  The slot ranges do not depend on p, so the first copies go out
// before pos is read; rows past p or past the CTA's range (which hold no
// position of this CTA's window and may hold anything) and the new slot's row
// are put right in shared memory once their sub-chunk has landed.  Each of
// the 4 warps takes 16 slots of a sub-chunk and keeps its own running max,
// sum and output for the (up to 16, zero-padded) query heads in registers,
// flash-attention style: scores q·Kᵀ and outputs P·V are bf16 tensor-core
// products (mma m16n8k16 with fp32 accumulation, fragments through ldmatrix
// from the swizzled tiles), P rounded to bf16 as in the prefill.  The sum of
// P comes out of the same product, from a column of ones beside V, so it adds
// exactly the rounded values that P·V adds.  The warps' states merge through
// shared memory at the end.
template <int HD> struct StepCfg {
  static constexpr int CH = HD <= 64 ? 128 : 64;   // smallest chunk (sizes the workspace)
  static constexpr int SC = 64;                    // slots per sub-chunk
  static constexpr int PW = HD < 64 ? HD : 64;     // panel width (elements): one TMA box row
  static constexpr int NPANEL = HD / PW;
  static constexpr int RB = PW * 2;                // bytes per panel row = swizzle span
  static constexpr int MAT_BYTES = SC * HD * 2;    // one matrix (K or V) of a sub-chunk
  static constexpr int STAGE_BYTES = 2 * MAT_BYTES;
  // Three stages at HD <= 64 keep the block at 52 KB, so that four CTAs fit
  // an SM and the split covers the batch in one wave with the work spread
  // more evenly over the SMs (four stages at three CTAs per SM measured
  // 15.2 us per step at 16 sequences, W = 2048, against 12.6 us).
  static constexpr int STG = HD <= 64 ? 3 : 2;
  static constexpr int CTAS_PER_SM = HD <= 64 ? 4 : 3;  // by shared memory
  static constexpr int KP = HD + 8;                // q tile pitch in bf16 (conflict-free ldmatrix)
  static constexpr int Q_OFF = STG * STAGE_BYTES;
  static constexpr int BAR_OFF = Q_OFF + 16 * KP * 2;
  static constexpr int SMEM = BAR_OFF + 64 + 1024;  // barriers, abort flag; 1024-byte alignment slack
  // after the main loop the stage buffers hold the merge: each warp's O
  // [4][16][HD] fp32, then the warps' max and sum [4][16] each
  static constexpr int WM_OFF = 4 * 16 * HD * 4;
  static_assert(WM_OFF + 2 * 4 * 16 * 4 <= Q_OFF, "merge fits the stage buffers");
  static_assert(STG * 8 + 8 <= 64, "barrier block");
  static constexpr int THREADS = 128;
};

// Byte offset of 16-byte chunk c (of HD / 8) in row r of a sub-chunk matrix
// as the tensor copy lays it out: NPANEL panels of [SC][RB], each row's
// chunks permuted by the swizzle of its span (128, 64 or 32 bytes).
template <int HD>
__device__ __forceinline__ uint32_t step_tile_off(int r, int c) {
  using Cfg = StepCfg<HD>;
  constexpr int CPR = Cfg::RB / 16;  // chunks per panel row
  const int panel = c / CPR, ci = c % CPR;
  int x;
  if constexpr (Cfg::RB == 128) x = ci ^ (r & 7);
  else if constexpr (Cfg::RB == 64) x = ci ^ ((r >> 1) & 3);
  else x = ci ^ ((r >> 2) & 1);
  return static_cast<uint32_t>(panel * Cfg::SC * Cfg::RB + r * Cfg::RB + x * 16);
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t saddr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(saddr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t saddr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(saddr));
}

template <int HD>
__global__ void __launch_bounds__(128) swa_step_split_kernel(
    const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
    const __nv_bfloat16* __restrict__ q_t, const __nv_bfloat16* __restrict__ k_t,
    const __nv_bfloat16* __restrict__ v_t, __nv_bfloat16* __restrict__ k_ring, __nv_bfloat16* __restrict__ v_ring,
    const int64_t* __restrict__ pos, float* __restrict__ ws, int Hq, int Hkv, int W, float scale_log2, int nsplit,
    int chunk) {
  using Cfg = StepCfg<HD>;
  constexpr int SC = Cfg::SC, KP = Cfg::KP, STG = Cfg::STG, RCH = HD / 8;
  extern __shared__ unsigned char sm_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
  __nv_bfloat16* Qs = reinterpret_cast<__nv_bfloat16*>(sm + Cfg::Q_OFF);     // [16][KP]
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + Cfg::BAR_OFF);            // [STG]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + STG);
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int group = Hq / Hkv;  // <= 16
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int j_lo = split * chunk;
  const int j_hi = static_cast<int64_t>(j_lo) + chunk < W ? j_lo + chunk : W;
  const int nsub = (j_hi - j_lo + SC - 1) / SC;
  const int64_t row_stride = static_cast<int64_t>(Hkv) * HD;           // elements between ring slots
  const int64_t noff = ((int64_t)b * Hkv + g) * HD;
  const uint32_t sm_base = smem_u32(sm);

  if (tid == 0) {
    for (int s = 0; s < STG; ++s) mbar_init(&full[s], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_launch_dependents();
  pdl_wait();  // q, k, v, the ring and pos all come from earlier kernels

  auto issue = [&](int stage, int sub) {  // one thread
    unsigned char* Ks = sm + stage * Cfg::STAGE_BYTES;
    unsigned char* Vs = Ks + Cfg::MAT_BYTES;
    const int j = j_lo + sub * SC;   // slots past W read as zeros
    mbar_arrive_expect_tx(&full[stage], Cfg::STAGE_BYTES);
#pragma unroll
    for (int pn = 0; pn < Cfg::NPANEL; ++pn) {
      tma_load_4d(Ks + pn * SC * Cfg::RB, &map_k, &full[stage], pn * Cfg::PW, g, j, b);
      tma_load_4d(Vs + pn * SC * Cfg::RB, &map_v, &full[stage], pn * Cfg::PW, g, j, b);
    }
  };
  if (tid == 0) {
    tma_prefetch_desc(&map_k);
    tma_prefetch_desc(&map_v);
    for (int st = 0; st < STG - 1 && st < nsub; ++st) issue(st, st);
  }

  const int64_t p = pos[b];
  const int jnew = static_cast<int>(p % W);
  // slots [j_lo, lim) of this CTA hold positions of the window
  const int lim = p + 1 < j_hi ? static_cast<int>(p + 1) : j_hi;
  for (int i = tid; i < 16 * RCH; i += 128) {
    const int hh = i / RCH, c = i % RCH;
    const uint4 v = hh < group ? reinterpret_cast<const uint4*>(q_t + ((int64_t)b * Hq + g * group + hh) * HD)[c]
                               : make_uint4(0u, 0u, 0u, 0u);
    reinterpret_cast<uint4*>(Qs + hh * KP)[c] = v;
  }
  if (jnew >= j_lo && jnew < j_hi && tid < RCH && SAMBA_CHECK(jnew >= 0 && jnew < W)) {  // the new key and value into their slot
    const int64_t roff = ((int64_t)b * W + jnew) * row_stride + (int64_t)g * HD;
    reinterpret_cast<uint4*>(k_ring + roff)[tid] = reinterpret_cast<const uint4*>(k_t + noff)[tid];
    reinterpret_cast<uint4*>(v_ring + roff)[tid] = reinterpret_cast<const uint4*>(v_t + noff)[tid];
  }

  uint32_t qa[HD / 16][4];
  float o[HD / 8][4], ol[4] = {0.f, 0.f, 0.f, 0.f};  // ol: P times a column of ones (the sums)
#pragma unroll
  for (int nt = 0; nt < HD / 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY;  // running max of rows gq and gq + 8, in log2 units
  constexpr uint32_t kOnes = 0x3F803F80u;  // two bf16 1.0
  bool ok = true;
  const int mi = lane >> 3, l7 = lane & 7;

  for (int sub = 0; sub < nsub; ++sub) {
    const int stage = sub % STG;
    ok = mbar_wait(&full[stage], (sub / STG) & 1, abort_flag) && ok;
    __syncthreads();
    unsigned char* Ks = sm + stage * Cfg::STAGE_BYTES;
    unsigned char* Vs = Ks + Cfg::MAT_BYTES;
    const int j0 = j_lo + sub * SC;
    // rows from lim on (past p, or past the CTA's range) become zeros and the
    // new slot's row becomes k_t, v_t
    const bool fix_tail = lim < j0 + SC;
    const bool fix_new = jnew >= j0 && jnew < j0 + SC && jnew < j_hi;
    if (fix_tail || fix_new) {  // uniform over the CTA
      for (int i = tid; i < SC * RCH; i += 128) {
        const int r = i / RCH, c = i % RCH, j = j0 + r;
        uint4* kd = reinterpret_cast<uint4*>(Ks + step_tile_off<HD>(r, c));
        uint4* vd = reinterpret_cast<uint4*>(Vs + step_tile_off<HD>(r, c));
        if (j == jnew) {
          *kd = reinterpret_cast<const uint4*>(k_t + noff)[c];
          *vd = reinterpret_cast<const uint4*>(v_t + noff)[c];
        } else if (j >= lim) {
          *kd = make_uint4(0u, 0u, 0u, 0u);
          *vd = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_shared();  // these writes come before the next tensor copy into the buffer
      __syncthreads();
    }
    if (sub == 0) {
#pragma unroll
      for (int ks = 0; ks < HD / 16; ++ks)
        ldsm_x4(qa[ks], smem_u32(Qs + ((mi & 1) * 8 + l7) * KP + 16 * ks + (mi >> 1) * 8));
    }
    const int r0 = 16 * warp;
    const uint32_t kb_base = sm_base + stage * Cfg::STAGE_BYTES, vb_base = kb_base + Cfg::MAT_BYTES;
    // scores S[head, slot] for this warp's 16 slots (two n8 tiles), raw
    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int ks = 0; ks < HD / 16; ++ks) {
      uint32_t kb[4];
      ldsm_x4(kb, kb_base + step_tile_off<HD>(r0 + (mi >> 1) * 8 + l7, 2 * ks + (mi & 1)));
      mma_bf16_16816(sc[0], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], kb[0], kb[1]);
      mma_bf16_16816(sc[1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], kb[2], kb[3]);
    }
    const int nval = lim - (j0 + r0);  // this warp's slots [0, nval) are in the window
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = 8 * nt + 2 * tq + (e & 1);
        sc[nt][e] = col < nval ? sc[nt][e] : -INFINITY;
        if (e < 2) mx0 = fmaxf(mx0, sc[nt][e]);
        else mx1 = fmaxf(mx1, sc[nt][e]);
      }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    // the scale is positive, so the max of the raw scores gives the max of
    // the scaled ones
    const float mn0 = fmaxf(m0, mx0 * scale_log2), mn1 = fmaxf(m1, mx1 * scale_log2);
    const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
    const float c0 = ex2_approx(m0 - mu0), c1 = ex2_approx(m1 - mu1);  // 0 while nothing was seen
    m0 = mn0;
    m1 = mn1;
    uint32_t pa[4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const __nv_bfloat162 lo = __floats2bfloat162_rn(ex2_approx(fmaf(sc[nt][0], scale_log2, -mu0)),
                                                       ex2_approx(fmaf(sc[nt][1], scale_log2, -mu0)));
      const __nv_bfloat162 hi = __floats2bfloat162_rn(ex2_approx(fmaf(sc[nt][2], scale_log2, -mu1)),
                                                       ex2_approx(fmaf(sc[nt][3], scale_log2, -mu1)));
      pa[2 * nt] = *reinterpret_cast<const uint32_t*>(&lo);
      pa[2 * nt + 1] = *reinterpret_cast<const uint32_t*>(&hi);
    }
    if (!__all_sync(0xffffffffu, c0 == 1.f && c1 == 1.f)) {  // a max moved: rescale
#pragma unroll
      for (int nt = 0; nt < HD / 8; ++nt) {
        o[nt][0] *= c0;
        o[nt][1] *= c0;
        o[nt][2] *= c1;
        o[nt][3] *= c1;
      }
      ol[0] *= c0;
      ol[1] *= c0;
      ol[2] *= c1;
      ol[3] *= c1;
    }
    // O[head, d] += P[head, slot] · V[slot, d]; A = P (k = slots 0-7 | 8-15)
#pragma unroll
    for (int jj = 0; jj < HD / 16; ++jj) {
      uint32_t vb[4];
      ldsm_x4_t(vb, vb_base + step_tile_off<HD>(r0 + (mi & 1) * 8 + l7, 2 * jj + (mi >> 1)));
      mma_bf16_16816(o[2 * jj], pa[0], pa[1], pa[2], pa[3], vb[0], vb[1]);
      mma_bf16_16816(o[2 * jj + 1], pa[0], pa[1], pa[2], pa[3], vb[2], vb[3]);
    }
    mma_bf16_16816(ol, pa[0], pa[1], pa[2], pa[3], kOnes, kOnes);
    // every warp has passed this iteration's barrier, so the buffer of the
    // previous sub-chunk is free for the one STG - 1 ahead
    if (tid == 0 && sub + STG - 1 < nsub) issue((sub + STG - 1) % STG, sub + STG - 1);
  }
  __syncthreads();  // the stage buffers now hold the merge (every copy has landed: each was waited for)

  // merge the four warps: per head M = max over warps, each warp's share
  // scaled by exp2(m_w - M) into its own slice (plain stores; shared-memory
  // atomics from the CTAs sharing an SM would serialise), the slices summed as the
  // partial is written
  float* Ow = reinterpret_cast<float*>(sm);                    // [4][16][HD]
  float* wm = reinterpret_cast<float*>(sm + Cfg::WM_OFF);      // [4][16]
  float* wl = wm + 64;                                         // [4][16]
  if (tq == 0) {
    wm[warp * 16 + gq] = m0;
    wm[warp * 16 + gq + 8] = m1;
    wl[warp * 16 + gq] = ol[0];
    wl[warp * 16 + gq + 8] = ol[2];
  }
  __syncthreads();
  float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    M0 = fmaxf(M0, wm[w * 16 + gq]);
    M1 = fmaxf(M1, wm[w * 16 + gq + 8]);
  }
  const float f0 = M0 == -INFINITY ? 0.f : ex2_approx(m0 - M0);
  const float f1 = M1 == -INFINITY ? 0.f : ex2_approx(m1 - M1);
  float* mine = Ow + warp * 16 * HD;
#pragma unroll
  for (int nt = 0; nt < HD / 8; ++nt) {
    const int col = 8 * nt + 2 * tq;
    *reinterpret_cast<float2*>(mine + gq * HD + col) = make_float2(o[nt][0] * f0, o[nt][1] * f0);
    *reinterpret_cast<float2*>(mine + (gq + 8) * HD + col) = make_float2(o[nt][2] * f1, o[nt][3] * f1);
  }
  if (!__syncthreads_and(ok)) return;  // a copy never landed: the status word says so
  for (int i = tid; i < group * HD; i += 128) {
    const int hh = i / HD, dd = i % HD;
    if (!SAMBA_CHECK(g * group + hh < Hq && split < nsplit && b < (int)gridDim.z)) continue;
    float* dst = ws + ((((int64_t)b * Hq + g * group + hh) * nsplit + split) * (HD + 2));
    dst[2 + dd] = Ow[hh * HD + dd] + Ow[(16 + hh) * HD + dd] + Ow[(32 + hh) * HD + dd] + Ow[(48 + hh) * HD + dd];
    if (dd == 0) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; ++w) M = fmaxf(M, wm[w * 16 + hh]);
      float l = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w)
        if (M != -INFINITY && wm[w * 16 + hh] != -INFINITY) l = fmaf(wl[w * 16 + hh], ex2_approx(wm[w * 16 + hh] - M), l);
      dst[0] = M;
      dst[1] = l;
    }
  }
}

template <int HD>
__global__ void swa_step_combine_kernel(const float* __restrict__ ws, __nv_bfloat16* __restrict__ o_t,
                                        int64_t* __restrict__ pos, int Hq, int nsplit) {
  pdl_launch_dependents();
  pdl_wait();
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
  if (!SAMBA_CHECK(hq < Hq && dd < HD && b < (int)gridDim.y)) return;
  o_t[((int64_t)b * Hq + hq) * HD + dd] = __float2bfloat16_rn(acc / l);
  if (hq == 0 && dd == 0) pos[b] += 1;
}

// Bytes of split partials: (max, sum, d outputs) per (batch, query head,
// split), for at most ceil(W / CH) splits.  SIZE_MAX when the product does
// not fit in size_t, so that no workspace (and no built-in scratch) is ever
// taken as large enough.
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

// Slots per CTA: as many splits as the CTAs an SM holds (ctas_per_sm) take
// over the batch and KV heads, at least 128 slots (so the partials fit the
// workspace size above, which counts splits of 128 slots, or 64 for
// d = 128) and a multiple of 64.
static int swa_step_chunk(int64_t B, int Hkv, int64_t W, int ctas_per_sm) {
  const int64_t per_split = static_cast<int64_t>(Hkv) * B;
  const int64_t target = std::max<int64_t>(1, ctas_per_sm * sm_count() / per_split);
  const int64_t c = (W + target - 1) / target;
  return static_cast<int>(std::max<int64_t>(128, (c + 63) / 64 * 64));
}

template <int HD>
static int swa_step_go(const void* q_t, const void* k_t, const void* v_t, void* k_ring, void* v_ring, int64_t* pos,
                       void* o_t, int64_t B, int Hq, int Hkv, int64_t W, float scale, void* ws, cudaStream_t s) {
  using Cfg = StepCfg<HD>;
  auto split_kern = swa_step_split_kernel<HD>;
  static PerDeviceOnce attr;
  const int arc = once_per_device(attr, [&] {
    return cudaFuncSetAttribute(split_kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM) == cudaSuccess
               ? SAMBA_OK
               : fail(SAMBA_ERR_CUDA, "samba_swa_step: cannot set shared memory size");
  });
  if (arc != SAMBA_OK) return arc;
  // the rings as [B][W][Hkv][d]; boxes of one panel x one head x 64 slots
  CUtensorMap mk, mv;
  const uint64_t dims[4] = {(uint64_t)HD, (uint64_t)Hkv, (uint64_t)W, (uint64_t)B};
  const uint64_t strides[3] = {(uint64_t)HD * 2, (uint64_t)Hkv * HD * 2, (uint64_t)W * Hkv * HD * 2};
  const uint32_t box[4] = {(uint32_t)Cfg::PW, 1u, (uint32_t)Cfg::SC, 1u};
  const CUtensorMapSwizzle sw = Cfg::RB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : (Cfg::RB == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  int rc = encode_tiled(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, k_ring, dims, strides, box, sw, "swa_step K ring");
  if (rc) return rc;
  rc = encode_tiled(&mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, v_ring, dims, strides, box, sw, "swa_step V ring");
  if (rc) return rc;
  const int chunk = swa_step_chunk(B, Hkv, W, Cfg::CTAS_PER_SM);
  const int nsplit = (int)((W + chunk - 1) / chunk);
  cudaError_t e = launch_pdl(split_kern, dim3(nsplit, Hkv, (unsigned)B), dim3(Cfg::THREADS), Cfg::SMEM, s, mk, mv,
                             reinterpret_cast<const __nv_bfloat16*>(q_t), reinterpret_cast<const __nv_bfloat16*>(k_t),
                             reinterpret_cast<const __nv_bfloat16*>(v_t), reinterpret_cast<__nv_bfloat16*>(k_ring),
                             reinterpret_cast<__nv_bfloat16*>(v_ring), (const int64_t*)pos,
                             reinterpret_cast<float*>(ws), Hq, Hkv, static_cast<int>(W), scale * 1.4426950408889634f,
                             nsplit, chunk);
  if (e != cudaSuccess) return fail(SAMBA_ERR_CUDA, "samba_swa_step: launch failed: %s", cudaGetErrorString(e));
  e = launch_pdl(swa_step_combine_kernel<HD>, dim3(Hq, (unsigned)B), dim3(HD), 0, s, (const float*)ws,
                 reinterpret_cast<__nv_bfloat16*>(o_t), pos, Hq, nsplit);
  if (e != cudaSuccess) return fail(SAMBA_ERR_CUDA, "samba_swa_step: launch failed: %s", cudaGetErrorString(e));
  return SAMBA_OK;
}

int launch_swa_step(const void* q_t, const void* k_t, const void* v_t, void* k_ring, void* v_ring, int64_t* pos,
                    void* o_t, int64_t B, int Hq, int Hkv, int d, int64_t W, float scale, void* ws, cudaStream_t s) {
  if (B > 65535) return fail(SAMBA_ERR_UNSUPPORTED, "samba_swa_step: batch too large");
  int rc;
  switch (d) {
    case 16: rc = swa_step_go<16>(q_t, k_t, v_t, k_ring, v_ring, pos, o_t, B, Hq, Hkv, W, scale, ws, s); break;
    case 32: rc = swa_step_go<32>(q_t, k_t, v_t, k_ring, v_ring, pos, o_t, B, Hq, Hkv, W, scale, ws, s); break;
    case 64: rc = swa_step_go<64>(q_t, k_t, v_t, k_ring, v_ring, pos, o_t, B, Hq, Hkv, W, scale, ws, s); break;
    default: rc = swa_step_go<128>(q_t, k_t, v_t, k_ring, v_ring, pos, o_t, B, Hq, Hkv, W, scale, ws, s); break;
  }
  if (rc != SAMBA_OK) return rc;
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

#ifdef SAMBA_DEBUG
// A store whose index is one past its 16-element buffer: the check skips it.
__device__ float g_check_buf[16];
__global__ void selftest_check_kernel(int i) {
  if (threadIdx.x == 0 && SAMBA_CHECK(i >= 0 && i < 16)) g_check_buf[i] = 1.f;
}
#endif

int launch_selftest_check(cudaStream_t s) {
#ifdef SAMBA_DEBUG
  selftest_check_kernel<<<1, 32, 0, s>>>(16);
  return check_launch("samba_selftest_check");
#else
  (void)s;
  return fail(SAMBA_ERR_UNSUPPORTED, "samba_selftest_check: the release build has no device-side checks");
#endif
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
