// Host-side helpers of the C ABI: error reporting, argument checks and TMA
// tensor-map encoding through the driver entry point (no link to libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdarg>
#include <algorithm>
#include <cstdio>
#include <mutex>
#include <string>

#include "../../include/samba.h"

namespace samba {

void set_error(const char* fmt, ...);
int fail(int code, const char* fmt, ...);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Checks a launch just issued; returns SAMBA_OK or SAMBA_ERR_CUDA.
int check_launch(const char* what);

// Encodes a tiled tensor map (row-major, dims[0] innermost, strides in bytes
// for dims 1..rank-1).  Returns SAMBA_OK or an error code (with the message set).
int encode_tiled(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                 const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                 CUtensorMapSwizzle swizzle, const char* what);

// Number of SMs of the current device.
int sm_count();

// Per-device one-time setup (function attributes apply to the device that is
// current when they are set).  once_per_device(o, f) runs f() unless it has
// already succeeded for the current device; thread-safe.
struct PerDeviceOnce {
  std::mutex mu;
  uint64_t done = 0;  // bit d: device d is set up
};
template <class F>
int once_per_device(PerDeviceOnce& o, F&& f) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(SAMBA_ERR_CUDA, "cannot query the current device");
  if (dev < 0 || dev >= 64) return f();  // no record past 64 devices: set up every time
  std::lock_guard<std::mutex> lock(o.mu);
  if ((o.done >> dev) & 1u) return SAMBA_OK;
  const int rc = f();
  if (rc == SAMBA_OK) o.done |= uint64_t(1) << dev;
  return rc;
}

// Per-translation-unit status readers (each kernel file keeps its own word).
int take_status_scan(cudaStream_t s);
int take_status_swa(cudaStream_t s);
int take_status_misc(cudaStream_t s);
int take_status_gemm(cudaStream_t s);
int launch_gemm(const samba_gemm_args& a, cudaStream_t stream);
int launch_selftest_check(cudaStream_t s);
size_t gemm_workspace_size(int64_t M, int64_t N);
size_t scan_bwd_workspace(int64_t B, int64_t L, int64_t D, int N);
int launch_scan_bwd(const samba_scan_bwd_args& a, cudaStream_t stream);
size_t swa_bwd_workspace(int64_t B, int64_t L, int Hq);
int launch_swa_bwd(const samba_swa_bwd_args& a, cudaStream_t stream);
int take_status_swa_bwd(cudaStream_t s);
int launch_selftest_wait(cudaStream_t s);

// Launchers (validated arguments only).
int launch_conv1d(const void* x, int x_dtype, const float* w, const float* bias, const float* cs_in, void* u,
                  int u_dtype, float* cs_out, int64_t B, int64_t L, int64_t D, int K, int silu,
                  cudaStream_t stream);
int launch_scan(const samba_scan_args& a, cudaStream_t stream);
int launch_swa(const samba_swa_args& a, cudaStream_t stream);
int launch_scan_step(float* h, float* conv_state, const void* x_t, int x_dtype, const void* z_t, int z_dtype,
                     const float* delta_t, const float* B_t, const float* C_t, const float* A, const float* Dskip,
                     const float* conv_w, const float* conv_b, void* y_t, int y_dtype, int64_t B, int64_t D,
                     int N, int K, uint32_t flags, cudaStream_t stream);
int launch_ring_fill(const void* k, const void* v, int64_t L, void* k_ring, void* v_ring, int64_t* pos, int64_t B,
                     int Hkv, int d, int64_t W, cudaStream_t stream);
size_t swa_step_workspace(int64_t B, int Hq, int d, int64_t W);
int launch_scan_carry(const float* h_in, const float* dsum, const float* A, const float* h_local, float* h_out,
                      int64_t B, int64_t D, int N, cudaStream_t stream);
int launch_conv_state(const void* x, int x_dtype, const float* cs_in, float* cs_out, int64_t B, int64_t L, int64_t D,
                      int K, cudaStream_t stream);
int launch_swa_step_noalloc(const void* q_t, const void* k_t, const void* v_t, void* k_ring, void* v_ring,
                            int64_t* pos, void* o_t, int64_t B, int Hq, int Hkv, int d, int64_t W, float scale,
                            cudaStream_t stream);
int launch_swa_step(const void* q_t, const void* k_t, const void* v_t, void* k_ring, void* v_ring, int64_t* pos,
                    void* o_t, int64_t B, int Hq, int Hkv, int d, int64_t W, float scale, void* ws,
                    cudaStream_t stream);

}  // namespace samba
