// Document-wise rotary positions and packed documents ("100 Millionen Token: Gedaechtnis
// oder Trugbild?", aitalk.it, section "Das Gehirn mit zwei Geschwindigkeiten": the
// position counter restarts at zero at the start of every document).
//
// msa_rope_docwise rotates q and k in place: dimensions i and i + d/2 of every head form
// a pair rotated by pos * theta_i, theta_i = base^(-2i/d), pos = the token's position in
// its own document.  It is an HBM-bound elementwise pass (read and write q and k once):
// a CTA takes kTokens consecutive tokens, computes their d/2 (cos, sin) pairs once into
// shared memory (angles in fp64, so positions up to 2^31 keep their full phase; sincos in
// fp64, rounded to fp32), then every thread rotates 16-byte chunks of the tokens' heads.
//
// msa_prefill_varlen_fwd runs the causal prefill on each packed document in turn
// (blocks restart at the document start; no selection or attention crosses a document
// boundary), with pointer offsets into the packed tensors.
#include <math.h>


#include "common.cuh"

namespace msa {
namespace {

constexpr int kRopeThreads = 256;
constexpr int kRopeTokens = 8;        // tokens per CTA iteration
constexpr int kMaxHalf = 64;          // d / 2

struct RopeArgs {
  double theta[kMaxHalf];
  int64_t n_tok;
  int hq, hkv, d, n_docs;
};

// Position of token t inside its document: cu[] holds the n_docs + 1 boundaries.
__device__ __forceinline__ int64_t doc_pos(const int32_t* __restrict__ cu, int n_docs, int64_t t) {
  int lo = 0, hi = n_docs;                 // largest doc with cu[doc] <= t
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)__ldg(cu + mid) <= t) lo = mid; else hi = mid;
  }
  return t - (int64_t)__ldg(cu + lo);
}

template <typename T>
__device__ __forceinline__ void rotate_chunk(T* __restrict__ row, int c, int half,
                                             const float* cs, const float* sn) {
  using V = Vec16<T>;
  constexpr int N = V::N;
  uint4* a = reinterpret_cast<uint4*>(row + c * N);
  uint4* b = reinterpret_cast<uint4*>(row + half + c * N);
  const uint4 ua = *a, ub = *b;
  float xa[N], xb[N];
  V::unpack(ua, xa);
  V::unpack(ub, xb);
  alignas(16) T ya[N];
  alignas(16) T yb[N];
#pragma unroll
  for (int e = 0; e < N; ++e) {
    const float c0 = cs[c * N + e], s0 = sn[c * N + e];
    ya[e] = from_f32<T>(xa[e] * c0 - xb[e] * s0);
    yb[e] = from_f32<T>(xb[e] * c0 + xa[e] * s0);
  }
  *a = *reinterpret_cast<const uint4*>(ya);
  *b = *reinterpret_cast<const uint4*>(yb);
}

template <typename T>
__global__ void __launch_bounds__(kRopeThreads)
rope_docwise_kernel(T* __restrict__ q, T* __restrict__ k, const int32_t* __restrict__ cu,
                    const __grid_constant__ RopeArgs a) {
  __shared__ float s_cos[kRopeTokens][kMaxHalf], s_sin[kRopeTokens][kMaxHalf];
  constexpr int N = Vec16<T>::N;
  const int half = a.d / 2;
  const int cpp = half / N;                          // 16-byte chunks per half head
  const int heads = a.hq + a.hkv;
  const int work = kRopeTokens * heads * cpp;
  for (int64_t t0 = (int64_t)blockIdx.x * kRopeTokens; t0 < a.n_tok;
       t0 += (int64_t)gridDim.x * kRopeTokens) {
    for (int i = threadIdx.x; i < kRopeTokens * half; i += kRopeThreads) {
      const int tt = i / half, f = i % half;
      const int64_t t = t0 + tt;
      if (t < a.n_tok) {
        const double ang = (double)doc_pos(cu, a.n_docs, t) * a.theta[f];
        double s, c;
        sincos(ang, &s, &c);
        s_cos[tt][f] = (float)c;
        s_sin[tt][f] = (float)s;
      }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < work; i += kRopeThreads) {
      const int tt = i / (heads * cpp);
      const int r = i - tt * heads * cpp;
      const int h = r / cpp, c = r - h * cpp;
      const int64_t t = t0 + tt;
      if (t >= a.n_tok) continue;
      T* row = h < a.hq ? q + (t * a.hq + h) * a.d : k + (t * a.hkv + (h - a.hq)) * a.d;
      rotate_chunk<T>(row, c, half, s_cos[tt], s_sin[tt]);
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_rope_docwise(const Shape& s, const int32_t* cu, int64_t n_docs, void* q,
                                void* k, double base, cudaStream_t st) {
  RopeArgs a{};
  const int half = (int)(s.d / 2);
  for (int i = 0; i < half; ++i) a.theta[i] = pow(base, -2.0 * i / (double)s.d);
  a.n_tok = s.batch * s.seq;
  a.hq = (int)s.hq;
  a.hkv = (int)s.hkv;
  a.d = (int)s.d;
  a.n_docs = (int)n_docs;
  const int64_t iters = (a.n_tok + kRopeTokens - 1) / kRopeTokens;
  const int64_t cap = (int64_t)sm_count() * 8;
  const unsigned grid = (unsigned)(iters < cap ? iters : cap);
  if (s.dtype == MSA_BF16)
    rope_docwise_kernel<__nv_bfloat16><<<grid, kRopeThreads, 0, st>>>(
        (__nv_bfloat16*)q, (__nv_bfloat16*)k, cu, a);
  else
    rope_docwise_kernel<float><<<grid, kRopeThreads, 0, st>>>((float*)q, (float*)k, cu, a);
  return cudaGetLastError();
}

}  // namespace msa
