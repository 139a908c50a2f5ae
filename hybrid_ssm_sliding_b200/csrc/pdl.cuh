// Programmatic dependent launch for the decode chain (projection GEMMs, the
// one-position conv, the scan step, the SWA step).
//
// A kernel launched with the programmatic-stream-serialization attribute may
// start while the kernel before it on the stream is still running, as soon as
// every CTA of that kernel has executed griddepcontrol.launch_dependents (or
// exited).  Its threads then call griddepcontrol.wait before touching anything
// the earlier kernel writes, which returns once that kernel has completed and
// its memory operations are visible.  Before the wait a kernel may only set up
// shared memory and tensor memory and read data no kernel of the chain writes
// (weights, tensor maps).  Launch latency and prologues then overlap the
// previous kernel's tail, and a projection can stream its first weight tiles
// before its input exists.
//
// Completion stays ordered along the chain: a kernel completes only after its
// own wait has returned, that is after its predecessor completed, so every
// earlier kernel has completed when a wait returns.  With the attribute off
// (SAMBA_NO_PDL set in the environment) the kernels launch plainly and the two
// instructions have nothing to wait for.
#pragma once

#include <cstdlib>

#include <cuda_runtime.h>

namespace samba {

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

inline bool pdl_enabled() {
  static const bool on = std::getenv("SAMBA_NO_PDL") == nullptr;
  return on;
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace samba
