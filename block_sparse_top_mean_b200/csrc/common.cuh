// Shared device helpers and internal launcher declarations of the msa library.
#pragma once

#include <cuda_bf16.h>
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/msa.h"

namespace msa {

constexpr int kWsHeader = 256;   // bytes at the start of every workspace (error word)
constexpr int kMaxTopk = 32;     // longest selection list a row can hold

__device__ __forceinline__ uint4 ldg16(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// Streaming 16-byte load that does not allocate in L1 (read-once data).
__device__ __forceinline__ uint4 ldg16_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ float bf16lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t w) {
  return __uint_as_float(w & 0xffff0000u);
}

// Unpacks 16 bytes of T into fp32 (exact for both types).
template <typename T> struct Vec16;
template <> struct Vec16<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void unpack(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
  }
};
template <> struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void unpack(const uint4& u, float* f) {
    f[0] = bf16lo_to_f32(u.x); f[1] = bf16hi_to_f32(u.x);
    f[2] = bf16lo_to_f32(u.y); f[3] = bf16hi_to_f32(u.y);
    f[4] = bf16lo_to_f32(u.z); f[5] = bf16hi_to_f32(u.z);
    f[6] = bf16lo_to_f32(u.w); f[7] = bf16hi_to_f32(u.w);
  }
};

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}
template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ void set_device_error(int* err, int bits) {
  if (err != nullptr) atomicOr(err, bits);
}

// ------------------------------------------------------------------ launchers
// All return cudaSuccess or the launch error; shapes are validated by the caller.

struct Shape {
  int64_t batch, seq, hq, hkv, d, block, topk, nb;
  float scale;
  int dtype;
};

cudaError_t launch_pool_keys(const Shape& s, const void* k, float* kbar, void* hi, void* lo,
                             int64_t n_seq, cudaStream_t st);

cudaError_t launch_block_scores(const Shape& s, const void* q, const float* kbar, float* scores,
                                cudaStream_t st);

// Causal prefill selection (fused scoring + top-k); writes idx [b, hkv, S, topk].
cudaError_t launch_topk_prefill(const Shape& s, const void* q, const float* kbar, int32_t* idx,
                                cudaStream_t st);
// The same selection restricted to the 64-token tiles whose flag byte is set.
cudaError_t launch_topk_prefill_flagged(const Shape& s, const void* q, const float* kbar,
                                        int32_t* idx, const uint8_t* flags, int flag_tile,
                                        cudaStream_t st);

// Decode selection: per-split candidate lists then a merge; writes idx [nq, hkv, topk].
size_t decode_select_ws_bytes(const Shape& s, int64_t n_query);
cudaError_t launch_topk_decode(const Shape& s, int64_t n_query, const void* q, const float* kbar,
                               int32_t* idx, void* ws, cudaStream_t st);

// Tensor-core decode selection (bf16 queries, d = 128); see topk_decode_tc.cu.  Needs the
// bank's pooled keys as bf16 hi/lo planes; workspace: per-CTA candidate lists.
bool tc_decode_supported(const Shape& s);
size_t topk_decode_tc_ws_bytes(const Shape& s, int64_t n_query);
// With `keys` given, writes instead of idx the best topk 64-bit keys per (query, group)
// [n_query, hkv, topk], sorted descending, block ids raised by block_offset (a shard of a
// bank reporting bank-wide ids).
cudaError_t launch_topk_decode_tc(const Shape& s, int64_t n_query, const void* q,
                                  const void* kbar_hi, const void* kbar_lo,
                                  const void* kbar_tiles, int32_t* idx, void* ws, int* err,
                                  cudaStream_t st, uint64_t* keys = nullptr,
                                  int64_t block_offset = 0);

// Memory Parallel decode (memory_parallel.cu): merge of the shards' key lists into the
// bank-wide selection and this shard's owned local ids; log-sum-exp combine of partials.
cudaError_t launch_merge_shard_keys(const uint64_t* keys, int64_t world, int64_t rows,
                                    int topk, int64_t block_begin, int64_t block_count,
                                    int32_t* idx, int32_t* idx_local, cudaStream_t st);
cudaError_t launch_combine_shards(const void* o_parts, const float* lse_parts, int64_t world,
                                  int64_t rows, int d, int dtype, void* o, float* lse,
                                  cudaStream_t st);

// Decode attention streamed through shared memory on mma.sync (bf16, d = 128,
// block % 64 == 0); see attn_decode_tc.cu.  Writes per-split partials (normalised O and
// lse, the same layout as the SIMT decode rows) for combine_splits_kernel.
bool tc_decode_attn_supported(const Shape& s);
int decode_attn_tc_nsplit(const Shape& s);
int decode_attn_tc_partials(const Shape& s);   // partials per (query, group)
cudaError_t launch_attn_decode_tc(const Shape& s, int64_t n_query, const void* q, const void* k,
                                  const void* v, const void* k_tiles, const void* v_tiles,
                                  const int32_t* idx, float* po, float* plse, int* err,
                                  cudaStream_t st);

// Encoded decode banks (bank_tiles.cu): K/V as per-head 64-key 16 KB tile images and
// pooled-key hi/lo planes as per-head 128-block 32 KB chunk images, both in the
// 128-byte-swizzled shared-memory layout the decode kernels consume.
size_t bank_kv_tiles_bytes(const Shape& s);
size_t bank_kbar_tiles_bytes(const Shape& s);
// One plane (hi or lo) of the encoded pooled keys; the image is the hi plane, the lo
// plane, then the selection bounds [2][hkv] fp32 (max ||lo_j||_2, max ||hi_j||_2 over the
// bank's blocks), padded to 256 bytes.
size_t bank_kbar_planes_bytes(const Shape& s);
constexpr int kMaxBoundGroups = 32;      // KV heads the bounds' 256 bytes hold
cudaError_t launch_encode_bank(const Shape& s, const void* k, const void* v, const void* kbar_hi,
                               const void* kbar_lo, void* k_tiles, void* v_tiles,
                               void* kbar_tiles, cudaStream_t st);

// Query-centric attention over selected blocks (SIMT, fp32 math).
size_t decode_attn_ws_bytes(const Shape& s, int64_t n_query);
cudaError_t launch_attn_prefill_rows(const Shape& s, const void* q, const void* k, const void* v,
                                     const int32_t* idx, void* o, float* lse, int* err,
                                     cudaStream_t st);
cudaError_t launch_attn_decode(const Shape& s, int64_t n_query, const void* q, const void* k,
                               const void* v, const void* k_tiles, const void* v_tiles,
                               const int32_t* idx, void* o, float* lse, void* ws, int* err,
                               cudaStream_t st);

// Backward of the key-centric tensor-core attention (attn_bwd_tc.cu): dq, dk, dv fp32.
bool tc_attn_bwd_supported(const Shape& s);
size_t tc_attn_bwd_ws_bytes(const Shape& s);       // recommended (one pass or 32 GiB slabs)
size_t tc_attn_bwd_ws_min_bytes(const Shape& s);   // one 2048-token slab
cudaError_t launch_attn_bwd_tc(const Shape& s, const void* q, const void* k, const void* v,
                               const void* o, const float* lse, const void* dout,
                               const int32_t* idx, float* dq, float* dk, float* dv, void* ws_body,
                               size_t ws_body_bytes, int* err, cudaStream_t st);

// Host-resident bank content (offload.cu): scratch of the staging step, and the step
// itself (marks the selected blocks, numbers them per group, gathers their K/V tiles
// from device-accessible host memory into an HBM staging bank and rewrites the selection
// as staging slots).
size_t offload_ws_bytes(const Shape& s, int64_t n_query, int tile_bytes);
cudaError_t launch_offload_stage(const Shape& s, int64_t n_query, const int32_t* idx,
                                 const void* k_host, const void* v_host, int tile_bytes,
                                 char* ws, int32_t** idx_staged_out, void** k_stage_out,
                                 void** v_stage_out, cudaStream_t st);

// Document-wise rotary positions (docs.cu): rotates q [T, hq, d] and k [T, hkv, d] in
// place, T = batch * seq packed tokens, positions from the device boundaries cu.
cudaError_t launch_rope_docwise(const Shape& s, const int32_t* cu, int64_t n_docs, void* q,
                                void* k, double base, cudaStream_t st);

// Host-side checks of a decode call's shapes and pointers (msa_api.cu), shared by the
// decode entry points; *empty is set for a call with no work, *tc when the tensor-core
// scan runs.  Touches no device state.
msa_status check_decode_args(const msa_params* p, int64_t n_query, const void* q,
                             const float* kbar, const void* kbar_hi, const void* kbar_lo,
                             const void* k_bank, const void* v_bank, const int32_t* idx,
                             const void* o, Shape* s, bool* tc, bool* empty);
size_t decode_ws_bytes(const Shape& s, int64_t n_query);   // header included

// Host helpers (host_util.cu): a 2-D bf16 TMA map over a row-major [rows, cols] tensor
// with 64-column x box_rows boxes and 128-byte swizzle; the device's SM count.
bool make_bf16_2d_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows);
int sm_count();

// Tensor-core prefill selection (bf16, d = 128); see topk_tc.cu.  Needs the pooled keys'
// bf16 hi/lo planes.
// A flag byte per (sequence, group, 64-token tile) marks tiles whose selection must be
// redone exactly by the SIMT kernel (launch_topk_prefill_flagged).
bool tc_topk_supported(const Shape& s);
size_t topk_tc_flag_bytes(const Shape& s);
cudaError_t launch_topk_prefill_tc(const Shape& s, const void* q, const float* kbar,
                                   const void* kbar_hi, const void* kbar_lo, int32_t* idx,
                                   uint8_t* flags, int* err, cudaStream_t st);

// Key-centric tensor-core attention (bf16, d = 128); see attn_tc.cu.
bool tc_attn_supported(const Shape& s);
size_t tc_attn_ws_bytes(const Shape& s);       // recommended (whole sequence or a 32 GiB slab)
size_t tc_attn_ws_min_bytes(const Shape& s);   // one 2048-token slab
int64_t tc_attn_slab_tokens(const Shape& s, size_t ws_body_bytes);   // 0: too small
// Runs in token slabs sized to the ws_body_bytes given (>= tc_attn_ws_min_bytes).
cudaError_t launch_attn_prefill_tc(const Shape& s, const void* q, const void* k, const void* v,
                                   const int32_t* idx, void* o, float* lse, void* ws_body,
                                   size_t ws_body_bytes, int* err, cudaStream_t st);

}  // namespace msa
