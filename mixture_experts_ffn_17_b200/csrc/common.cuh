// common.cuh -- small device helpers shared by the kernels of this library.
#pragma once

#include <cstdint>
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

}  // namespace moe
