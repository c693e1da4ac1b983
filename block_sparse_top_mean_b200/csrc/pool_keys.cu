// Step 1: pooled routing key per KV block (mean of the block's keys, per KV head).
//
// HBM-streaming kernel: one CTA per (sequence, block); each thread owns one 16-byte
// column vector of the [hkv * d] token row and walks the block's tokens in order, so a
// warp reads 512 contiguous bytes per token and every byte of K is read exactly once.
// Accumulation is fp32 in token order, then one IEEE division by the token count.
#include "common.cuh"

namespace msa {
namespace {

constexpr int kPoolThreads = 128;
constexpr int kPoolUnroll = 8;

template <typename T>
__global__ void __launch_bounds__(kPoolThreads)
pool_keys_kernel(const T* __restrict__ k, float* __restrict__ kbar,
                 __nv_bfloat16* __restrict__ hi, __nv_bfloat16* __restrict__ lo, int64_t S,
                 int64_t nb, int row_elems, int64_t block) {
  constexpr int V = Vec16<T>::N;
  const int64_t j = blockIdx.x;
  const int64_t b = blockIdx.y;
  const int64_t t0 = j * block;
  const int64_t t1 = (t0 + block < S) ? t0 + block : S;
  const int nvec = row_elems / V;
  for (int vi = threadIdx.x; vi < nvec; vi += blockDim.x) {
    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
    const T* base = k + (b * S + t0) * (int64_t)row_elems + (int64_t)vi * V;
    int64_t t = t0;
    for (; t + kPoolUnroll <= t1; t += kPoolUnroll) {
      uint4 x[kPoolUnroll];
#pragma unroll
      for (int u = 0; u < kPoolUnroll; ++u)
        x[u] = ldg16_stream(base + (t - t0 + u) * (int64_t)row_elems);
#pragma unroll
      for (int u = 0; u < kPoolUnroll; ++u) {
        float f[V];
        Vec16<T>::unpack(x[u], f);
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] += f[e];
      }
    }
    for (; t < t1; ++t) {
      float f[V];
      Vec16<T>::unpack(ldg16_stream(base + (t - t0) * (int64_t)row_elems), f);
#pragma unroll
      for (int e = 0; e < V; ++e) acc[e] += f[e];
    }
    const float n = (float)(t1 - t0);
    const int64_t o = (b * nb + j) * (int64_t)row_elems + (int64_t)vi * V;
    float m[V];
#pragma unroll
    for (int e = 0; e < V; ++e) m[e] = acc[e] / n;
#pragma unroll
    for (int e = 0; e < V; e += 4)
      *reinterpret_cast<float4*>(kbar + o + e) = make_float4(m[e], m[e + 1], m[e + 2], m[e + 3]);
    if (hi != nullptr || lo != nullptr) {
#pragma unroll
      for (int e = 0; e < V; ++e) {
        const __nv_bfloat16 h = __float2bfloat16_rn(m[e]);
        if (hi != nullptr) hi[o + e] = h;
        if (lo != nullptr) lo[o + e] = __float2bfloat16_rn(m[e] - __bfloat162float(h));
      }
    }
  }
}

}  // namespace

cudaError_t launch_pool_keys(const Shape& s, const void* k, float* kbar, void* hi, void* lo,
                             int64_t n_seq, cudaStream_t st) {
  const int row = (int)(s.hkv * s.d);
  dim3 grid((unsigned)s.nb, (unsigned)n_seq);
  if (s.dtype == MSA_BF16) {
    pool_keys_kernel<__nv_bfloat16><<<grid, kPoolThreads, 0, st>>>(
        (const __nv_bfloat16*)k, kbar, (__nv_bfloat16*)hi, (__nv_bfloat16*)lo, s.seq, s.nb, row,
        s.block);
  } else {
    pool_keys_kernel<float><<<grid, kPoolThreads, 0, st>>>(
        (const float*)k, kbar, (__nv_bfloat16*)hi, (__nv_bfloat16*)lo, s.seq, s.nb, row, s.block);
  }
  return cudaGetLastError();
}

}  // namespace msa
