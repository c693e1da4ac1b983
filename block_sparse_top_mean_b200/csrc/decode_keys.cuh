// 64-bit selection keys of the decode scan: the order-preserving bits of an fp32 score
// above the complement of the block index, so one unsigned comparison implements
// (score descending, block index ascending); key 0 is "empty" and below every key.
#pragma once

#include <math_constants.h>
#include <stdint.h>

namespace msa {
namespace keys {

// Order-preserving unsigned bits of a (finite) score; 0 is below every score.
__device__ __forceinline__ uint32_t score_ord(float s) {
  const uint32_t b = __float_as_uint(s + 0.0f);            // -0 -> +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float ord_score(uint32_t ord) {
  if (ord == 0u) return -CUDART_INF_F;
  return __uint_as_float((ord & 0x80000000u) ? (ord & 0x7fffffffu) : ~ord);
}
__device__ __forceinline__ uint64_t make_key(float s, int64_t j) {
  return ((uint64_t)score_ord(s) << 32) | (uint32_t)(~(uint32_t)j);
}
__device__ __forceinline__ float key_score(uint64_t key) {   // -inf for an empty entry
  return ord_score((uint32_t)(key >> 32));
}
__device__ __forceinline__ int key_block(uint64_t key) {
  return (int)(~(uint32_t)key);
}

__device__ __forceinline__ uint64_t umax64(uint64_t a, uint64_t b) { return a > b ? a : b; }
__device__ __forceinline__ uint64_t umin64(uint64_t a, uint64_t b) { return a < b ? a : b; }

// y, x sorted descending over lanes -> the 32 largest of both, sorted descending.
__device__ __forceinline__ uint64_t warp_merge_desc(uint64_t y, uint64_t x, int lane) {
  uint64_t z = umax64(y, __shfl_sync(0xffffffffu, x, 31 - lane));
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
    const uint64_t p = __shfl_xor_sync(0xffffffffu, z, j);
    z = ((lane & j) == 0) ? umax64(z, p) : umin64(z, p);
  }
  return z;
}

// Descending bitonic merge of a 64-key list held as (z0, z1): lane l holds ranks l and
// 32 + l of a bitonic sequence; afterwards they hold ranks l and 32 + l sorted.
__device__ __forceinline__ void warp_sort_bitonic64(uint64_t& z0, uint64_t& z1, int lane) {
  const uint64_t a = umax64(z0, z1), b = umin64(z0, z1);
  z0 = a;
  z1 = b;
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
    const uint64_t p0 = __shfl_xor_sync(0xffffffffu, z0, j);
    const uint64_t p1 = __shfl_xor_sync(0xffffffffu, z1, j);
    const bool lower = (lane & j) == 0;
    z0 = lower ? umax64(z0, p0) : umin64(z0, p0);
    z1 = lower ? umax64(z1, p1) : umin64(z1, p1);
  }
}

}  // namespace keys
}  // namespace msa
