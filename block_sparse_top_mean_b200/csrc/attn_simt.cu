// Step 4, query-centric SIMT form: exact softmax attention over the selected blocks.
//
// One warp per (row, split), where a row is one (token, GQA group) in prefill or one
// (query, group) in decode; the warp serves all G query heads of the group, which share
// the selection.  Keys are taken 32 at a time (one key per lane for the q.k dots, with
// the group's queries broadcast from shared memory), then an online softmax in base 2
// (logits pre-multiplied by scale*log2(e)) and the P.V update with each lane owning d/32
// output dimensions.  All math is fp32.  This is the fp32-input path and the decode
// path (memory-bound: every selected K/V byte is read once per row).
#include <math_constants.h>

#include "common.cuh"

namespace msa {
namespace {

constexpr int kWarps = 4;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct RowsArgs {
  const void* q; const void* k; const void* v; const int32_t* idx;
  void* o; float* lse;           // final outputs (when nsplit == 1)
  float* po; float* plse;        // partials (when nsplit > 1)
  int* err;
  int64_t n_rows;                // prefill: b*hkv*S ; decode: nq*hkv
  int64_t S, nb, block;
  int hq, hkv, topk, nsplit, slots_per_split;
  float scale_log2;
  int causal;                    // 1 = prefill rows, 0 = decode rows
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(kWarps * 32)
attn_rows_kernel(RowsArgs a) {
  constexpr int DPL = D / 32;          // output dims per lane
  constexpr int V = Vec16<T>::N;
  __shared__ __align__(16) float qsm[kWarps][G][D];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t task = (int64_t)blockIdx.x * kWarps + warp;
  if (task >= a.n_rows * a.nsplit) return;
  const int64_t row = task / a.nsplit;
  const int split = (int)(task % a.nsplit);

  // Row geometry.
  int64_t b = 0, t = 0, g, qoff, koff_b;   // koff_b: element offset of (b, p=0, g)
  if (a.causal) {
    t = row % a.S;
    g = (row / a.S) % a.hkv;
    b = row / (a.S * a.hkv);
    qoff = ((b * a.S + t) * a.hq + g * G) * (int64_t)D;
    koff_b = (b * a.S * a.hkv + g) * (int64_t)D;
  } else {
    g = row % a.hkv;
    const int64_t n = row / a.hkv;
    qoff = (n * a.hq + g * G) * (int64_t)D;
    koff_b = g * (int64_t)D;
  }
  const T* Q = reinterpret_cast<const T*>(a.q);
  const T* K = reinterpret_cast<const T*>(a.k);
  const T* Vv = reinterpret_cast<const T*>(a.v);
  const int64_t kstride = (int64_t)a.hkv * D;   // elements between consecutive tokens

#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < DPL; ++e)
      qsm[warp][h][lane * DPL + e] = to_f32<T>(Q[qoff + (int64_t)h * D + lane * DPL + e]);
  __syncwarp();

  float m[G], l[G], acc[G][DPL];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -CUDART_INF_F; l[h] = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[h][e] = 0.f;
  }

  const int32_t* irow = a.idx + row * (int64_t)a.topk;
  const int64_t own = a.causal ? t / a.block : -1;
  const int s0 = split * a.slots_per_split;
  const int s1 = min(a.topk, s0 + a.slots_per_split);
  for (int s = s0; s < s1; ++s) {
    const int64_t j = irow[s];
    if (j == -1) continue;
    if (j < -1 || j >= a.nb || (a.causal && j > own)) {
      if (lane == 0) set_device_error(a.err, MSA_DEVERR_IDX_RANGE);
      continue;
    }
    const int64_t p_lo = j * a.block;
    int64_t p_hi = p_lo + a.block < a.S ? p_lo + a.block : a.S;
    if (a.causal && j == own) p_hi = t + 1;
    for (int64_t pc = p_lo; pc < p_hi; pc += 32) {
      const int64_t p = pc + lane;
      const bool valid = p < p_hi;
      float dot[G];
#pragma unroll
      for (int h = 0; h < G; ++h) dot[h] = 0.f;
      if (valid) {
        const T* kr = K + koff_b + p * kstride;
#pragma unroll 4
        for (int c = 0; c < D / V; ++c) {
          float f[V];
          Vec16<T>::unpack(ldg16(kr + c * V), f);
#pragma unroll
          for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < V; ++e) dot[h] = fmaf(qsm[warp][h][c * V + e], f[e], dot[h]);
        }
      }
      float pr[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float s2 = valid ? dot[h] * a.scale_log2 : -CUDART_INF_F;
        const float mn = fmaxf(m[h], warp_max(s2));
        const float alpha = exp2f(m[h] - mn);
        pr[h] = exp2f(s2 - mn);
        l[h] = l[h] * alpha + pr[h];
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[h][e] *= alpha;
        m[h] = mn;
      }
      const int nk = (int)((p_hi - pc) < 32 ? (p_hi - pc) : 32);
      for (int kk = 0; kk < nk; ++kk) {
        const T* vr = Vv + koff_b + (pc + kk) * kstride + lane * DPL;
        float vf[DPL];
#pragma unroll
        for (int e = 0; e < DPL; ++e) vf[e] = to_f32<T>(vr[e]);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float pk = __shfl_sync(0xffffffffu, pr[h], kk);
#pragma unroll
          for (int e = 0; e < DPL; ++e) acc[h][e] = fmaf(pk, vf[e], acc[h][e]);
        }
      }
    }
  }

#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float lt = warp_sum(l[h]);
    const float inv = lt > 0.f ? 1.f / lt : 0.f;
    const float lse_h = lt > 0.f ? (m[h] + log2f(lt)) * kLn2 : -CUDART_INF_F;
    if (a.nsplit == 1) {
      T* O = reinterpret_cast<T*>(a.o);
#pragma unroll
      for (int e = 0; e < DPL; ++e)
        O[qoff + (int64_t)h * D + lane * DPL + e] = from_f32<T>(acc[h][e] * inv);
      if (a.lse != nullptr && lane == 0) {
        if (a.causal)
          a.lse[(b * a.hq + g * G + h) * a.S + t] = lse_h;
        else
          a.lse[qoff / D + h] = lse_h;
      }
    } else {
      const int64_t pr_i = (row * a.nsplit + split) * G + h;
#pragma unroll
      for (int e = 0; e < DPL; ++e) a.po[pr_i * D + lane * DPL + e] = acc[h][e] * inv;
      if (lane == 0) a.plse[pr_i] = lse_h;
    }
  }
}

// Merges split partials (O_s normalised, lse_s): O = sum_s w_s O_s / sum_s w_s with
// w_s = exp(lse_s - max lse).  One warp per (row, head).
template <typename T, int D>
__global__ void combine_splits_kernel(const float* __restrict__ po, const float* __restrict__ plse,
                                      T* __restrict__ o, float* __restrict__ lse, int64_t n_rows,
                                      int G, int nsplit, int hkv, int hq) {
  constexpr int DPL = D / 32;
  const int64_t task = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (task >= n_rows * G) return;
  const int64_t row = task / G;
  const int h = (int)(task % G);
  float mx = -CUDART_INF_F;
  for (int s = 0; s < nsplit; ++s) mx = fmaxf(mx, plse[(row * nsplit + s) * G + h]);
  float acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
  float den = 0.f;
  if (mx > -CUDART_INF_F) {
    for (int s = 0; s < nsplit; ++s) {
      const int64_t pi = (row * nsplit + s) * G + h;
      const float w = exp2f((plse[pi] - mx) * kLog2e);
      den += w;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = fmaf(w, po[pi * D + lane * DPL + e], acc[e]);
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  // decode rows: row = n*hkv + g -> output head (n, g*G + h)
  const int64_t n = row / hkv, g = row % hkv;
  const int64_t oh = n * hq + g * G + h;
#pragma unroll
  for (int e = 0; e < DPL; ++e) o[oh * D + lane * DPL + e] = from_f32<T>(acc[e] * inv);
  if (lse != nullptr && lane == 0) lse[oh] = den > 0.f ? mx + logf(den) : -CUDART_INF_F;
}

constexpr int kDecodeSplitSlots = 4;   // selected blocks per decode warp

template <typename T, int D, int G>
cudaError_t run_rows(const RowsArgs& a, cudaStream_t st) {
  const int64_t tasks = a.n_rows * a.nsplit;
  const int64_t grid = (tasks + kWarps - 1) / kWarps;
  attn_rows_kernel<T, D, G><<<(unsigned)grid, kWarps * 32, 0, st>>>(a);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t dispatch_g(int G, const RowsArgs& a, cudaStream_t st) {
  switch (G) {
    case 1: return run_rows<T, D, 1>(a, st);
    case 2: return run_rows<T, D, 2>(a, st);
    case 4: return run_rows<T, D, 4>(a, st);
    case 8: return run_rows<T, D, 8>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t dispatch(const Shape& s, const RowsArgs& a, cudaStream_t st) {
  const int G = (int)(s.hq / s.hkv);
  if (s.dtype == MSA_BF16)
    return s.d == 128 ? dispatch_g<__nv_bfloat16, 128>(G, a, st)
                      : dispatch_g<__nv_bfloat16, 64>(G, a, st);
  return s.d == 128 ? dispatch_g<float, 128>(G, a, st) : dispatch_g<float, 64>(G, a, st);
}

RowsArgs base_args(const Shape& s) {
  RowsArgs a{};
  a.S = s.seq; a.nb = s.nb; a.block = s.block;
  a.hq = (int)s.hq; a.hkv = (int)s.hkv; a.topk = (int)s.topk;
  a.scale_log2 = s.scale * kLog2e;
  return a;
}

int decode_nsplit_attn(const Shape& s) {
  return (int)((s.topk + kDecodeSplitSlots - 1) / kDecodeSplitSlots);
}

}  // namespace

cudaError_t launch_attn_prefill_rows(const Shape& s, const void* q, const void* k, const void* v,
                                     const int32_t* idx, void* o, float* lse, int* err,
                                     cudaStream_t st) {
  RowsArgs a = base_args(s);
  a.q = q; a.k = k; a.v = v; a.idx = idx; a.o = o; a.lse = lse; a.err = err;
  a.n_rows = s.batch * s.hkv * s.seq;
  a.nsplit = 1; a.slots_per_split = (int)s.topk; a.causal = 1;
  return dispatch(s, a, st);
}

// Partials per (query, group): the SIMT rows write one per split, the streamed kernel one
// per split and consumer warp.
int decode_partials(const Shape& s) {
  return tc_decode_attn_supported(s) ? decode_attn_tc_partials(s) : decode_nsplit_attn(s);
}

size_t decode_attn_ws_bytes(const Shape& s, int64_t n_query) {
  const int G = (int)(s.hq / s.hkv);
  const size_t np = (size_t)n_query * s.hkv * decode_partials(s) * G;
  return ((np * s.d * sizeof(float) + 255) / 256) * 256 + np * sizeof(float) + 256;
}

cudaError_t launch_attn_decode(const Shape& s, int64_t n_query, const void* q, const void* k,
                               const void* v, const void* k_tiles, const void* v_tiles,
                               const int32_t* idx, void* o, float* lse, void* ws, int* err,
                               cudaStream_t st) {
  RowsArgs a = base_args(s);
  const int G = (int)(s.hq / s.hkv);
  a.q = q; a.k = k; a.v = v; a.idx = idx; a.err = err;
  a.n_rows = n_query * s.hkv;
  a.nsplit = decode_nsplit_attn(s); a.slots_per_split = kDecodeSplitSlots; a.causal = 0;
  const bool tc = tc_decode_attn_supported(s);
  const int nparts = tc ? decode_attn_tc_partials(s) : a.nsplit;
  const size_t np = (size_t)a.n_rows * nparts * G;
  a.po = reinterpret_cast<float*>(ws);
  a.plse = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) +
                                    ((np * s.d * sizeof(float) + 255) / 256) * 256);
  if (k_tiles != nullptr && !tc) return cudaErrorInvalidValue;   // encoded banks: tc only
  if (a.nsplit == 1 && !tc) { a.o = o; a.lse = lse; }
  cudaError_t e = tc ? launch_attn_decode_tc(s, n_query, q, k, v, k_tiles, v_tiles, idx, a.po,
                                             a.plse, err, st)
                     : dispatch(s, a, st);
  if (e != cudaSuccess || (a.nsplit == 1 && !tc)) return e;
  const int64_t tasks = a.n_rows * G;
  const unsigned grid = (unsigned)((tasks + 3) / 4);
  if (s.dtype == MSA_BF16) {
    if (s.d == 128)
      combine_splits_kernel<__nv_bfloat16, 128><<<grid, 128, 0, st>>>(
          a.po, a.plse, (__nv_bfloat16*)o, lse, a.n_rows, G, nparts, (int)s.hkv, (int)s.hq);
    else
      combine_splits_kernel<__nv_bfloat16, 64><<<grid, 128, 0, st>>>(
          a.po, a.plse, (__nv_bfloat16*)o, lse, a.n_rows, G, nparts, (int)s.hkv, (int)s.hq);
  } else {
    if (s.d == 128)
      combine_splits_kernel<float, 128><<<grid, 128, 0, st>>>(
          a.po, a.plse, (float*)o, lse, a.n_rows, G, nparts, (int)s.hkv, (int)s.hq);
    else
      combine_splits_kernel<float, 64><<<grid, 128, 0, st>>>(
          a.po, a.plse, (float*)o, lse, a.n_rows, G, nparts, (int)s.hkv, (int)s.hq);
  }
  return cudaGetLastError();
}

}  // namespace msa
