// Steps 2+3: index-branch scores against the pooled keys and top-k block selection.
//
// Per CTA: a tile of kRows query rows of one GQA group.  The group-summed queries
// (sum over the group's heads, fp32) and chunks of kChunk pooled keys sit transposed in
// shared memory; 256 threads compute the kRows x kChunk score tile with a 4x4 register
// micro-tile each (exact fp32 FMA chain over d), and one thread per row folds the tile
// into that row's running top list.  Blocks are visited in ascending order, so a strict
// "greater than the current worst" insert keeps the lower block index on ties, and the
// evicted entry is the worst one (lowest score, highest index on ties).  The score
// matrix never leaves shared memory.
//
// Prefill (causal): rows are tokens; eligible blocks are j < t/block; the own block is
// added at the end.  Decode: rows are queries, every block is eligible, CTAs split the
// bank's blocks and emit per-split candidate lists that a merge kernel reduces.
#include <math_constants.h>

#include "common.cuh"

namespace msa {
namespace {

constexpr int kRows = 64;
constexpr int kChunk = 64;
constexpr int kThreads = 256;
constexpr int kPadR = kRows + 4;
constexpr int kPadC = kChunk + 4;

template <int D>
struct TopkSmem {
  float qsT[D][kPadR];
  float kbT[D][kPadC];
  float sc[kRows][kChunk + 1];
  float lsc[kRows][kMaxTopk];
  int lidx[kRows][kMaxTopk];
};

struct RowList {
  int cnt, worst;
  float worst_s;
  int worst_j;
};

__device__ __forceinline__ void recompute_worst(RowList& L, const float* ls, const int* li) {
  int w = 0;
  float ws = ls[0];
  int wj = li[0];
  for (int e = 1; e < L.cnt; ++e) {
    const float s = ls[e];
    const int j = li[e];
    if (s < ws || (s == ws && j > wj)) { w = e; ws = s; wj = j; }
  }
  L.worst = w; L.worst_s = ws; L.worst_j = wj;
}

__device__ __forceinline__ void list_insert(RowList& L, int n_take, float s, int j, float* ls,
                                            int* li) {
  if (L.cnt < n_take) {
    ls[L.cnt] = s; li[L.cnt] = j; ++L.cnt;
    if (L.cnt == n_take) recompute_worst(L, ls, li);
  } else if (n_take > 0 && s > L.worst_s) {
    ls[L.worst] = s; li[L.worst] = j;
    recompute_worst(L, ls, li);
  }
}

template <typename T, int D>
__device__ __forceinline__ void load_group_qsum(TopkSmem<D>& sm, const T* q, int64_t row0,
                                                int64_t n_rows, int64_t row_stride, int G) {
  // q row r: q + (row0 + r) * row_stride, G heads of D consecutive elements each.
  for (int e = threadIdx.x; e < kRows * D; e += kThreads) {
    const int r = e / D, dd = e % D;
    float acc = 0.f;
    if (row0 + r < n_rows) {
      const T* p = q + (row0 + r) * row_stride + dd;
      for (int h = 0; h < G; ++h) acc += to_f32<T>(p[(int64_t)h * D]);
    }
    sm.qsT[dd][r] = acc;
  }
}

template <int D>
__device__ __forceinline__ void load_kbar_chunk(TopkSmem<D>& sm, const float* kb, int64_t j0,
                                                int64_t jend, int64_t j_stride) {
  // kb + j * j_stride is block j's pooled key for this group (D floats).
  for (int e = threadIdx.x; e < kChunk * D; e += kThreads) {
    const int c = e / D, dd = e % D;
    sm.kbT[dd][c] = (j0 + c < jend) ? kb[(j0 + c) * j_stride + dd] : 0.f;
  }
}

template <int D>
__device__ __forceinline__ void score_tile(TopkSmem<D>& sm) {
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
#pragma unroll 8
  for (int dd = 0; dd < D; ++dd) {
    const float4 qa = *reinterpret_cast<const float4*>(&sm.qsT[dd][ty * 4]);
    const float4 kb = *reinterpret_cast<const float4*>(&sm.kbT[dd][tx * 4]);
    const float qv[4] = {qa.x, qa.y, qa.z, qa.w};
    const float kv[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(qv[a], kv[c], acc[a][c]);
  }
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) sm.sc[ty * 4 + a][tx * 4 + c] = acc[a][c];
}

// ---------------------------------------------------------------- prefill (causal)
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
topk_prefill_kernel(const T* __restrict__ q, const float* __restrict__ kbar,
                    int32_t* __restrict__ idx, int64_t S, int64_t nb, int hq, int hkv,
                    int64_t block, int topk, const uint8_t* __restrict__ only) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  TopkSmem<D>& sm = *reinterpret_cast<TopkSmem<D>*>(smem_raw);
  const int64_t t0 = (int64_t)blockIdx.x * kRows;
  const int g = blockIdx.y;
  const int64_t b = blockIdx.z;
  // restricted run: only the tiles flagged by the tensor-core selection
  if (only != nullptr && only[((int64_t)b * hkv + g) * gridDim.x + blockIdx.x] == 0) return;
  const int G = hq / hkv;
  const int r = threadIdx.x;
  // rows of this tile: tokens t0 .. t0+kRows-1 of sequence b, group g
  load_group_qsum<T, D>(sm, q + (b * S) * hq * (int64_t)D + (int64_t)g * G * D, t0, S,
                        (int64_t)hq * D, G);
  const int64_t t_last = (t0 + kRows <= S ? t0 + kRows : S) - 1;
  const int64_t jmax = t_last / block;  // blocks [0, jmax) can be eligible for some row
  const int64_t own = (r < kRows && t0 + r < S) ? (t0 + r) / block : 0;
  const int n_take = (int)((own < topk - 1) ? own : topk - 1);
  RowList L{0, 0, -CUDART_INF_F, -1};
  const float* kb = kbar + (b * nb) * hkv * (int64_t)D + (int64_t)g * D;
  for (int64_t j0 = 0; j0 < jmax; j0 += kChunk) {
    __syncthreads();
    load_kbar_chunk<D>(sm, kb, j0, jmax, (int64_t)hkv * D);
    __syncthreads();
    score_tile<D>(sm);
    __syncthreads();
    if (r < kRows && t0 + r < S) {
      const int64_t cend = (own - j0 < kChunk) ? own - j0 : kChunk;
      for (int c = 0; c < cend; ++c) list_insert(L, n_take, sm.sc[r][c], (int)(j0 + c),
                                                 sm.lsc[r], sm.lidx[r]);
    }
  }
  if (r < kRows && t0 + r < S) {
    int* li = sm.lidx[r];
    li[L.cnt] = (int)own;
    const int n = L.cnt + 1;
    for (int a = 1; a < n; ++a) {  // insertion sort by block index
      const int x = li[a];
      int c = a - 1;
      while (c >= 0 && li[c] > x) { li[c + 1] = li[c]; --c; }
      li[c + 1] = x;
    }
    int32_t* out = idx + ((b * hkv + g) * S + t0 + r) * (int64_t)topk;
    for (int e = 0; e < topk; ++e) out[e] = (e < n) ? li[e] : -1;
  }
}

// ---------------------------------------------------------------- decode (bank scan)
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
topk_decode_split_kernel(const T* __restrict__ q, const float* __restrict__ kbar,
                         float* __restrict__ cand_s, int32_t* __restrict__ cand_j,
                         int64_t n_query, int64_t nb, int hq, int hkv, int topk,
                         int64_t per_split) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  TopkSmem<D>& sm = *reinterpret_cast<TopkSmem<D>*>(smem_raw);
  const int split = blockIdx.x;
  const int g = blockIdx.y;
  const int64_t n0 = (int64_t)blockIdx.z * kRows;
  const int G = hq / hkv;
  const int r = threadIdx.x;
  load_group_qsum<T, D>(sm, q + (int64_t)g * G * D, n0, n_query, (int64_t)hq * D, G);
  const int64_t jb = (int64_t)split * per_split;
  const int64_t je = (jb + per_split < nb) ? jb + per_split : nb;
  RowList L{0, 0, -CUDART_INF_F, -1};
  const float* kb = kbar + (int64_t)g * D;
  for (int64_t j0 = jb; j0 < je; j0 += kChunk) {
    __syncthreads();
    load_kbar_chunk<D>(sm, kb, j0, je, (int64_t)hkv * D);
    __syncthreads();
    score_tile<D>(sm);
    __syncthreads();
    if (r < kRows) {
      const int64_t cend = (je - j0 < kChunk) ? je - j0 : kChunk;
      for (int c = 0; c < cend; ++c)
        list_insert(L, topk, sm.sc[r][c], (int)(j0 + c), sm.lsc[r], sm.lidx[r]);
    }
  }
  if (r < kRows && n0 + r < n_query) {
    // candidates of (query n, group g, split): [n][g][split][topk]
    const int64_t nsplit = gridDim.x;
    const int64_t o = (((n0 + r) * hkv + g) * nsplit + split) * (int64_t)topk;
    for (int e = 0; e < topk; ++e) {
      cand_s[o + e] = (e < L.cnt) ? sm.lsc[r][e] : -CUDART_INF_F;
      cand_j[o + e] = (e < L.cnt) ? sm.lidx[r][e] : -1;
    }
  }
}

// One warp per (query, group): exact top-k of the union of the split lists under
// (score desc, index asc), written ascending.
__global__ void topk_decode_merge_kernel(const float* __restrict__ cand_s,
                                         const int32_t* __restrict__ cand_j,
                                         int32_t* __restrict__ idx, int nsplit, int topk) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int n_c = nsplit * topk;
  float* cs = reinterpret_cast<float*>(smem_raw);
  int* cj = reinterpret_cast<int*>(cs + n_c);
  __shared__ int chosen[kMaxTopk];
  const int64_t row = blockIdx.x;
  const int lane = threadIdx.x;
  for (int e = lane; e < n_c; e += 32) {
    cs[e] = cand_s[row * n_c + e];
    cj[e] = cand_j[row * n_c + e];
  }
  __syncwarp();
  int n_chosen = 0;
  for (int k = 0; k < topk; ++k) {
    float bs = -CUDART_INF_F;
    int bj = -1, bp = -1;
    for (int e = lane; e < n_c; e += 32) {
      const int j = cj[e];
      if (j < 0) continue;
      const float s = cs[e];
      if (bj < 0 || s > bs || (s == bs && j < bj)) { bs = s; bj = j; bp = e; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, bs, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      const int op = __shfl_xor_sync(0xffffffffu, bp, o);
      if (oj >= 0 && (bj < 0 || os > bs || (os == bs && oj < bj))) { bs = os; bj = oj; bp = op; }
    }
    if (bj < 0) break;
    if (lane == 0) { chosen[k] = bj; cj[bp] = -1; }
    ++n_chosen;
    __syncwarp();
  }
  if (lane == 0) {
    for (int a = 1; a < n_chosen; ++a) {
      const int x = chosen[a];
      int c = a - 1;
      while (c >= 0 && chosen[c] > x) { chosen[c + 1] = chosen[c]; --c; }
      chosen[c + 1] = x;
    }
    for (int e = 0; e < topk; ++e) idx[row * topk + e] = (e < n_chosen) ? chosen[e] : -1;
  }
}

// ---------------------------------------------------------------- materialised scores
template <typename T>
__global__ void block_scores_kernel(const T* __restrict__ q, const float* __restrict__ kbar,
                                    float* __restrict__ scores, int64_t S, int64_t nb, int hq,
                                    int hkv, int D, int64_t block, int64_t total) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= total) return;
  const int64_t j = e % nb;
  const int64_t t = (e / nb) % S;
  const int64_t g = (e / (nb * S)) % hkv;
  const int64_t b = e / (nb * S * hkv);
  if (j >= t / block) { scores[e] = -CUDART_INF_F; return; }
  const int G = hq / hkv;
  const T* qp = q + ((b * S + t) * hq + g * G) * (int64_t)D;
  const float* kp = kbar + ((b * nb + j) * hkv + g) * (int64_t)D;
  float acc = 0.f;
  for (int dd = 0; dd < D; ++dd) {
    float qs = 0.f;
    for (int h = 0; h < G; ++h) qs += to_f32<T>(qp[(int64_t)h * D + dd]);
    acc = fmaf(qs, kp[dd], acc);
  }
  scores[e] = acc;
}

template <typename KernelT>
cudaError_t set_smem(KernelT k, size_t bytes) {
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

int decode_nsplit(const Shape& s) {
  // ~2 CTAs per SM over all groups, at least one chunk of blocks per split
  int64_t want = (2 * 148 + s.hkv - 1) / s.hkv;
  int64_t max_split = (s.nb + kChunk - 1) / kChunk;
  if (want > max_split) want = max_split;
  if (want < 1) want = 1;
  return (int)want;
}

}  // namespace

cudaError_t launch_block_scores(const Shape& s, const void* q, const float* kbar, float* scores,
                                cudaStream_t st) {
  const int64_t total = s.batch * s.hkv * s.seq * s.nb;
  if (total == 0) return cudaSuccess;
  const int64_t blocks = (total + 255) / 256;
  if (s.dtype == MSA_BF16)
    block_scores_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(
        (const __nv_bfloat16*)q, kbar, scores, s.seq, s.nb, (int)s.hq, (int)s.hkv, (int)s.d,
        s.block, total);
  else
    block_scores_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(
        (const float*)q, kbar, scores, s.seq, s.nb, (int)s.hq, (int)s.hkv, (int)s.d, s.block,
        total);
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t topk_prefill_t(const Shape& s, const void* q, const float* kbar, int32_t* idx,
                                  cudaStream_t st, const uint8_t* only = nullptr) {
  const size_t smem = sizeof(TopkSmem<D>);
  cudaError_t e = set_smem(topk_prefill_kernel<T, D>, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((s.seq + kRows - 1) / kRows), (unsigned)s.hkv, (unsigned)s.batch);
  topk_prefill_kernel<T, D><<<grid, kThreads, smem, st>>>((const T*)q, kbar, idx, s.seq, s.nb,
                                                          (int)s.hq, (int)s.hkv, s.block,
                                                          (int)s.topk, only);
  return cudaGetLastError();
}

cudaError_t launch_topk_prefill(const Shape& s, const void* q, const float* kbar, int32_t* idx,
                                cudaStream_t st) {
  if (s.dtype == MSA_BF16)
    return s.d == 128 ? topk_prefill_t<__nv_bfloat16, 128>(s, q, kbar, idx, st)
                      : topk_prefill_t<__nv_bfloat16, 64>(s, q, kbar, idx, st);
  return s.d == 128 ? topk_prefill_t<float, 128>(s, q, kbar, idx, st)
                    : topk_prefill_t<float, 64>(s, q, kbar, idx, st);
}

cudaError_t launch_topk_prefill_flagged(const Shape& s, const void* q, const float* kbar,
                                        int32_t* idx, const uint8_t* flags, int flag_tile,
                                        cudaStream_t st) {
  if (flag_tile != kRows) return cudaErrorInvalidValue;   // one flag per SIMT tile
  if (s.dtype == MSA_BF16)
    return s.d == 128 ? topk_prefill_t<__nv_bfloat16, 128>(s, q, kbar, idx, st, flags)
                      : topk_prefill_t<__nv_bfloat16, 64>(s, q, kbar, idx, st, flags);
  return s.d == 128 ? topk_prefill_t<float, 128>(s, q, kbar, idx, st, flags)
                    : topk_prefill_t<float, 64>(s, q, kbar, idx, st, flags);
}

size_t decode_select_ws_bytes(const Shape& s, int64_t n_query) {
  const size_t n = (size_t)n_query * s.hkv * decode_nsplit(s) * s.topk;
  return n * (sizeof(float) + sizeof(int32_t)) + 256;
}

template <typename T, int D>
static cudaError_t topk_decode_t(const Shape& s, int64_t n_query, const void* q,
                                 const float* kbar, int32_t* idx, void* ws, cudaStream_t st) {
  const int nsplit = decode_nsplit(s);
  const int64_t per_split = (s.nb + nsplit - 1) / nsplit;
  const size_t n = (size_t)n_query * s.hkv * nsplit * s.topk;
  float* cs = reinterpret_cast<float*>(ws);
  int32_t* cj = reinterpret_cast<int32_t*>(
      reinterpret_cast<char*>(ws) + ((n * sizeof(float) + 255) / 256) * 256);
  const size_t smem = sizeof(TopkSmem<D>);
  cudaError_t e = set_smem(topk_decode_split_kernel<T, D>, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)nsplit, (unsigned)s.hkv, (unsigned)((n_query + kRows - 1) / kRows));
  topk_decode_split_kernel<T, D><<<grid, kThreads, smem, st>>>(
      (const T*)q, kbar, cs, cj, n_query, s.nb, (int)s.hq, (int)s.hkv, (int)s.topk, per_split);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t msmem = (size_t)nsplit * s.topk * (sizeof(float) + sizeof(int));
  if ((e = set_smem(topk_decode_merge_kernel, msmem)) != cudaSuccess) return e;
  topk_decode_merge_kernel<<<(unsigned)(n_query * s.hkv), 32, msmem, st>>>(cs, cj, idx, nsplit,
                                                                          (int)s.topk);
  return cudaGetLastError();
}

cudaError_t launch_topk_decode(const Shape& s, int64_t n_query, const void* q, const float* kbar,
                               int32_t* idx, void* ws, cudaStream_t st) {
  if (s.dtype == MSA_BF16)
    return s.d == 128 ? topk_decode_t<__nv_bfloat16, 128>(s, n_query, q, kbar, idx, ws, st)
                      : topk_decode_t<__nv_bfloat16, 64>(s, n_query, q, kbar, idx, ws, st);
  return s.d == 128 ? topk_decode_t<float, 128>(s, n_query, q, kbar, idx, ws, st)
                    : topk_decode_t<float, 64>(s, n_query, q, kbar, idx, ws, st);
}

}  // namespace msa
