// Memory Parallel decode ("100 Millionen Token: Gedaechtnis oder Trugbild?", aitalk.it,
// section "Das Gehirn mit zwei Geschwindigkeiten": each GPU holds part of the routing
// keys, the queries are broadcast, the relevance scores are aggregated, and only the
// selected documents are loaded).
//
// A bank is split into contiguous block ranges, one per rank.  Each rank scans its own
// range (the tensor-core decode scan, keys with bank-wide block ids), the ranks exchange
// their top-k keys per (query, group) (an all-gather of world x n_query x hkv x topk
// 64-bit keys), and every rank merges them here into the bank-wide selection: exactly
// the unsharded top-k, because each block of the bank-wide top-k is in the top-k of its
// own shard.  A rank then attends only the selected blocks it owns (the others are -1 in
// its local list) and the ranks' partial outputs, each normalised with its log-sum-exp,
// are combined by combine_shards_kernel into the softmax over the whole selection.
#include <math_constants.h>

#include "common.cuh"
#include "decode_keys.cuh"

namespace msa {
namespace {

using namespace keys;

constexpr float kLog2e = 1.4426950408889634f;

// One warp per (query, group) row: lists of `topk` keys sorted descending, one per rank.
__global__ void merge_shard_keys_kernel(const uint64_t* __restrict__ keys, int64_t world,
                                        int64_t rows, int topk, int64_t block_begin,
                                        int64_t block_count, int32_t* __restrict__ idx,
                                        int32_t* __restrict__ idx_local) {
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (w >= rows) return;
  uint64_t y = 0ull;
  for (int64_t r = 0; r < world; ++r) {                // rank order: a fixed merge order
    const uint64_t x = lane < topk ? __ldg(keys + (r * rows + w) * topk + lane) : 0ull;
    y = warp_merge_desc(y, x, lane);
  }
  int j = (lane < topk && y != 0ull) ? key_block(y) : 0x7fffffff;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {                  // ascending block ids, empties last
#pragma unroll
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      const int p = __shfl_xor_sync(0xffffffffu, j, jj);
      const bool take_min = ((lane & jj) == 0) == ((lane & k) == 0);
      j = take_min ? min(j, p) : max(j, p);
    }
  }
  if (lane < topk) {
    const bool empty = j == 0x7fffffff;
    idx[w * topk + lane] = empty ? -1 : j;
    const bool own = !empty && j >= block_begin && j < block_begin + block_count;
    if (idx_local != nullptr) idx_local[w * topk + lane] = own ? (int)(j - block_begin) : -1;
  }
}

// One warp per (query, head): O = sum_r w_r O_r / sum_r w_r, w_r = exp(lse_r - max lse),
// lse = max + log sum_r w_r; ranks without a selected block (lse_r = -inf) weigh 0.
template <typename T, int D>
__global__ void combine_shards_kernel(const T* __restrict__ o_parts,
                                      const float* __restrict__ lse_parts, int64_t world,
                                      int64_t rows, T* __restrict__ o, float* __restrict__ lse) {
  constexpr int DPL = D / 32;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (w >= rows) return;
  float mx = -CUDART_INF_F;
  for (int64_t r = 0; r < world; ++r) mx = fmaxf(mx, __ldg(lse_parts + r * rows + w));
  float acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  float den = 0.f;
  if (mx > -CUDART_INF_F) {
    for (int64_t r = 0; r < world; ++r) {
      const float l = __ldg(lse_parts + r * rows + w);
      if (!(l > -CUDART_INF_F)) continue;
      const float wt = exp2f((l - mx) * kLog2e);
      den += wt;
      const T* src = o_parts + (r * rows + w) * D + lane * DPL;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = fmaf(wt, to_f32<T>(src[e]), acc[e]);
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
  for (int e = 0; e < DPL; ++e) o[w * D + lane * DPL + e] = from_f32<T>(acc[e] * inv);
  if (lse != nullptr && lane == 0) lse[w] = den > 0.f ? mx + logf(den) : -CUDART_INF_F;
}

}  // namespace

cudaError_t launch_merge_shard_keys(const uint64_t* keys, int64_t world, int64_t rows,
                                    int topk, int64_t block_begin, int64_t block_count,
                                    int32_t* idx, int32_t* idx_local, cudaStream_t st) {
  merge_shard_keys_kernel<<<(unsigned)((rows + 3) / 4), 128, 0, st>>>(
      keys, world, rows, topk, block_begin, block_count, idx, idx_local);
  return cudaGetLastError();
}

cudaError_t launch_combine_shards(const void* o_parts, const float* lse_parts, int64_t world,
                                  int64_t rows, int d, int dtype, void* o, float* lse,
                                  cudaStream_t st) {
  const unsigned grid = (unsigned)((rows + 3) / 4);
  if (dtype == MSA_BF16) {
    if (d == 128)
      combine_shards_kernel<__nv_bfloat16, 128><<<grid, 128, 0, st>>>(
          (const __nv_bfloat16*)o_parts, lse_parts, world, rows, (__nv_bfloat16*)o, lse);
    else
      combine_shards_kernel<__nv_bfloat16, 64><<<grid, 128, 0, st>>>(
          (const __nv_bfloat16*)o_parts, lse_parts, world, rows, (__nv_bfloat16*)o, lse);
  } else {
    if (d == 128)
      combine_shards_kernel<float, 128><<<grid, 128, 0, st>>>(
          (const float*)o_parts, lse_parts, world, rows, (float*)o, lse);
    else
      combine_shards_kernel<float, 64><<<grid, 128, 0, st>>>(
          (const float*)o_parts, lse_parts, world, rows, (float*)o, lse);
  }
  return cudaGetLastError();
}

}  // namespace msa
