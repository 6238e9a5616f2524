// common.cuh -- small device helpers shared by the kernels of this library.
#pragma once

#include <cstdint>
#include <utility>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace moe {

// Raise an error bit in the device status word and the CTA's abort flag.
__device__ __forceinline__ void raise_status(uint32_t* status, volatile uint32_t* abort_flag, uint32_t bit) {
  if (status) atomicOr(status, bit);
  if (abort_flag) *abort_flag = 1u;
}

__device__ __forceinline__ uint8_t* align_1024(uint8_t* p) {
  uint32_t s = ptx::smem_u32(p);
  uint32_t pad = (1024u - (s & 1023u)) & 1023u;
  return p + pad;
}

// (value, index) ordering of every top-k here: larger value first, on equal
// values the lower index first.
__device__ __forceinline__ bool key_before(float va, int ia, float vb, int ib) {
  return (va > vb) || (va == vb && ia < ib);
}

// Programmatic dependent launch.  The kernels of one forward pass are
// launched with programmatic stream serialisation, so the next kernel may be
// scheduled while this one runs and do its prologue (barrier init, TMEM
// allocation, descriptor prefetch) early.  grid_dependency_wait() returns once
// the previous kernel in the stream has completed and its writes are visible
// (at once when the launch carried no such attribute); every kernel calls it
// before it touches memory an earlier kernel wrote, and before any early
// return, so completion of a kernel implies completion of all earlier ones.
// Then it allows the next kernel to be scheduled.
#ifndef MOE_PDL
#define MOE_PDL 1
#endif

__device__ __forceinline__ void grid_dependency_wait() {
#if MOE_PDL
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif
}

template <typename... K, typename... A>
cudaError_t launch_chained(void (*kernel)(K...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                           A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = MOE_PDL ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

}  // namespace moe
