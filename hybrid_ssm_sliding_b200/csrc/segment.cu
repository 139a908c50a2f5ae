// Joining scan segments: the carry of the selective-scan state from one
// segment of a sequence to the next (samba_scan_carry), and the conv state a
// segment hands on (samba_conv_state).
//
// Page "SAMBA混合注意力状态空间模型", section 数学框架 / Mamba层: the state
// follows h_t = Ā_t h_{t-1} + B̄_t x_t with Ā_t = exp(Δ_t A).  Over a segment
// the map from its start state to its end state is affine with slope
// Π_t exp(Δ_t A) = exp(A Σ_t Δ_t), so a segment scanned from zero joins its
// predecessor through one exp per (channel, state).
#include "common.cuh"
#include "host.hpp"

namespace samba {

__device__ __forceinline__ float seg_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// h_out = exp(A dsum) h_in + h_local; one thread per (b, c, n), the exp as
// 2^(A log2e · dsum) like the scan's decays.
__global__ void scan_carry_kernel(const float* __restrict__ h_in, const float* __restrict__ dsum,
                                  const float* __restrict__ A, const float* __restrict__ h_local,
                                  float* __restrict__ h_out, int64_t B, int64_t D, int N) {
  const int64_t total = B * D * N;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t bc = e / N;          // b * D + c
    const int64_t c = bc % D;
    const int n = (int)(e % N);
    const float decay = seg_ex2((A[c * N + n] * 1.4426950408889634f) * dsum[bc]);
    const float start = h_in ? h_in[e] : 0.f;
    h_out[e] = fmaf(decay, start, h_local[e]);
  }
}

int launch_scan_carry(const float* h_in, const float* dsum, const float* A, const float* h_local, float* h_out,
                      int64_t B, int64_t D, int N, cudaStream_t s) {
  const int64_t total = B * D * N;
  const int blocks = (int)std::min<int64_t>((total + 255) / 256, (int64_t)sm_count() * 8);
  scan_carry_kernel<<<blocks, 256, 0, s>>>(h_in, dsum, A, h_local, h_out, B, D, N);
  return check_launch("samba_scan_carry");
}

// conv_state_out[b, c, j] = entry L + j - (K-1) of (conv_state_in, x).
template <typename XT>
__global__ void seg_conv_state_kernel(const XT* __restrict__ x, const float* __restrict__ cs_in,
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

int launch_conv_state(const void* x, int x_dtype, const float* cs_in, float* cs_out, int64_t B, int64_t L, int64_t D,
                      int K, cudaStream_t s) {
  const int64_t n = B * D * (K - 1);
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 4096));
  if (x_dtype == SAMBA_BF16)
    seg_conv_state_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16*>(x), cs_in,
                                                                 cs_out, B, L, D, K);
  else
    seg_conv_state_kernel<float><<<blocks, 256, 0, s>>>(reinterpret_cast<const float*>(x), cs_in, cs_out, B, L, D, K);
  return check_launch("samba_conv_state");
}

}  // namespace samba
