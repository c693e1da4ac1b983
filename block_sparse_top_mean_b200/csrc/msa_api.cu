// C ABI of the msa library: host-side argument checks, workspace layout, launches.
// Every check runs before any CUDA call, so a rejected call touches no device state.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "common.cuh"

using msa::Shape;

namespace {

constexpr int64_t kMaxElems = (int64_t)1 << 40;   // guards every size product below
constexpr int kTileBytesKV = 16384;                // one encoded 64-key K or V tile

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }
size_t round256(size_t x) { return (x + 255) / 256 * 256; }
int* err_word(void* ws) { return reinterpret_cast<int*>(ws); }
char* ws_body(void* ws) { return reinterpret_cast<char*>(ws) + msa::kWsHeader; }

// Shape checks shared by every entry point.  `bank` = decode (seq is bank tokens).
msa_status check_params(const msa_params* p, bool bank, Shape* s) {
  if (p == nullptr) return MSA_ERR_INVALID_ARG;
  if (p->batch < 0 || p->seq < 0 || p->hq < 1 || p->hkv < 1 || p->d < 1 || p->block < 1 ||
      p->topk < 1)
    return MSA_ERR_INVALID_ARG;
  if (p->hq % p->hkv != 0) return MSA_ERR_INVALID_ARG;
  if (!isfinite(p->scale)) return MSA_ERR_INVALID_ARG;
  if (p->dtype != MSA_F32 && p->dtype != MSA_BF16) return MSA_ERR_INVALID_ARG;
  if (p->d != 64 && p->d != 128) return MSA_ERR_UNSUPPORTED;
  const int64_t G = p->hq / p->hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return MSA_ERR_UNSUPPORTED;
  if (p->topk > msa::kMaxTopk) return MSA_ERR_UNSUPPORTED;
  if (p->hkv > 65535) return MSA_ERR_UNSUPPORTED;
  const int64_t bsz = bank ? 1 : p->batch;
  if (bsz > 65535) return MSA_ERR_UNSUPPORTED;
  if (p->seq > kMaxElems / (p->hq * p->d) || (bsz > 0 && p->seq * p->hq * p->d > kMaxElems / bsz))
    return MSA_ERR_UNSUPPORTED;
  s->batch = bsz; s->seq = p->seq; s->hq = p->hq; s->hkv = p->hkv; s->d = p->d;
  s->block = p->block; s->topk = p->topk; s->scale = p->scale; s->dtype = p->dtype;
  s->nb = (p->seq + p->block - 1) / p->block;
  if (s->nb > INT32_MAX / 2) return MSA_ERR_UNSUPPORTED;
  return MSA_OK;
}

bool empty_prefill(const Shape& s) { return s.batch == 0 || s.seq == 0; }

size_t kbar_bytes(const Shape& s) { return (size_t)s.batch * s.nb * s.hkv * s.d * sizeof(float); }
// Fallback flags of the tensor-core selection (one byte per 64-token tile).
size_t topk_flag_ws(const Shape& s) {
  return msa::tc_topk_supported(s) ? round256(msa::topk_tc_flag_bytes(s)) : 0;
}
// bf16 hi or lo plane of the pooled keys; only the tensor-core selection uses them.
size_t kbar_split_bytes(const Shape& s) {
  return msa::tc_topk_supported(s) ? (size_t)s.batch * s.nb * s.hkv * s.d * 2 : 0;
}

// Decode selection scratch: enough for the SIMT scan and, where it applies, the
// tensor-core scan (which of the two runs depends on the planes the caller passes).
size_t decode_sel_ws(const Shape& s, int64_t n_query) {
  size_t n = msa::decode_select_ws_bytes(s, n_query);
  if (msa::tc_decode_supported(s)) {
    const size_t t = msa::topk_decode_tc_ws_bytes(s, n_query);
    if (t > n) n = t;
  }
  return n;
}

// Attention scratch: the recommended size, or the smallest the tensor-core path accepts
// (it then walks the sequence in more, smaller token slabs).
size_t attn_ws(const Shape& s, bool minimum) {
  if (!msa::tc_attn_supported(s)) return 0;
  return round256(minimum ? msa::tc_attn_ws_min_bytes(s) : msa::tc_attn_ws_bytes(s));
}

// Bytes of the prefill workspace in front of the attention scratch.
size_t prefill_fixed_ws(const Shape& s) {
  return round256(kbar_bytes(s)) + 2 * round256(kbar_split_bytes(s)) + topk_flag_ws(s);
}

size_t ws_bytes_for(const Shape& s, int op, int64_t n_query) {
  switch (op) {
    case MSA_OP_TOPK_SELECT:
      return msa::kWsHeader + topk_flag_ws(s);
    case MSA_OP_SPARSE_ATTN:
    case MSA_OP_SPARSE_ATTN_MIN:
      return msa::kWsHeader + attn_ws(s, op == MSA_OP_SPARSE_ATTN_MIN);
    case MSA_OP_PREFILL:
    case MSA_OP_PREFILL_MIN:
      return msa::kWsHeader + prefill_fixed_ws(s) + attn_ws(s, op == MSA_OP_PREFILL_MIN);
    case MSA_OP_DECODE:
      return msa::kWsHeader + round256(decode_sel_ws(s, n_query)) +
             round256(msa::decode_attn_ws_bytes(s, n_query));
    case MSA_OP_SPARSE_ATTN_BWD:
    case MSA_OP_SPARSE_ATTN_BWD_MIN:
      if (!msa::tc_attn_bwd_supported(s)) return 0;
      return msa::kWsHeader + round256(op == MSA_OP_SPARSE_ATTN_BWD_MIN
                                           ? msa::tc_attn_bwd_ws_min_bytes(s)
                                           : msa::tc_attn_bwd_ws_bytes(s));
    case MSA_OP_DECODE_OFFLOAD:
      return msa::kWsHeader + round256(decode_sel_ws(s, n_query)) +
             round256(msa::decode_attn_ws_bytes(s, n_query)) +
             round256(msa::offload_ws_bytes(s, n_query, kTileBytesKV));
    default:
      return 0;
  }
}

// The attention-bearing calls accept anything from the minimum size up.
msa_status check_ws(const Shape& s, int op, int64_t n_query, const void* ws, size_t ws_bytes) {
  if (op == MSA_OP_SPARSE_ATTN) op = MSA_OP_SPARSE_ATTN_MIN;
  if (op == MSA_OP_PREFILL) op = MSA_OP_PREFILL_MIN;
  if (op == MSA_OP_SPARSE_ATTN_BWD) op = MSA_OP_SPARSE_ATTN_BWD_MIN;
  const size_t need = ws_bytes_for(s, op, n_query);
  if (ws == nullptr || ws_bytes < need || !aligned256(ws)) return MSA_ERR_WORKSPACE;
  return MSA_OK;
}

msa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MSA_OK : MSA_ERR_CUDA; }

// bf16 with d = 128 and the split planes present runs the tensor-core selection;
// otherwise the fp32 SIMT one.
cudaError_t launch_selection(const Shape& s, const void* q, const float* kbar,
                             const void* kbar_hi, const void* kbar_lo, int32_t* idx,
                             uint8_t* flags, int* err, cudaStream_t st) {
  if (kbar_hi != nullptr && kbar_lo != nullptr && msa::tc_topk_supported(s))
    return msa::launch_topk_prefill_tc(s, q, kbar, kbar_hi, kbar_lo, idx, flags, err, st);
  return msa::launch_topk_prefill(s, q, kbar, idx, st);
}

// bf16 with d = 128 and 128-multiple blocks runs on the tensor cores (key-centric tiles);
// everything else on the query-centric SIMT kernel.
cudaError_t launch_attention(const Shape& s, const void* q, const void* k, const void* v,
                             const int32_t* idx, void* o, float* lse, char* scratch,
                             size_t scratch_bytes, int* err, cudaStream_t st) {
  if (msa::tc_attn_supported(s))
    return msa::launch_attn_prefill_tc(s, q, k, v, idx, o, lse, scratch, scratch_bytes, err, st);
  return msa::launch_attn_prefill_rows(s, q, k, v, idx, o, lse, err, st);
}


}  // namespace

namespace msa {

msa_status check_decode_args(const msa_params* p, int64_t n_query, const void* q,
                             const float* kbar, const void* kbar_hi, const void* kbar_lo,
                             const void* k_bank, const void* v_bank, const int32_t* idx,
                             const void* o, Shape* s, bool* tc, bool* empty) {
  *tc = false;
  *empty = false;
  msa_status st = check_params(p, true, s);
  if (st != MSA_OK) return st;
  if (n_query < 0) return MSA_ERR_INVALID_ARG;
  if (n_query == 0 || s->seq == 0) {
    *empty = true;
    return MSA_OK;
  }
  if (n_query > 65535 * 64) return MSA_ERR_UNSUPPORTED;
  // the tensor-core scan reads the bf16 planes; the SIMT scan the fp32 pooled keys
  *tc = kbar_hi != nullptr && kbar_lo != nullptr && msa::tc_decode_supported(*s);
  if (q == nullptr || (!*tc && kbar == nullptr) || k_bank == nullptr || v_bank == nullptr ||
      idx == nullptr || o == nullptr)
    return MSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kbar) || !aligned16(kbar_hi) || !aligned16(kbar_lo) ||
      !aligned16(k_bank) || !aligned16(v_bank) || !aligned16(o))
    return MSA_ERR_INVALID_ARG;
  return MSA_OK;
}

size_t decode_ws_bytes(const Shape& s, int64_t n_query) {
  return ws_bytes_for(s, MSA_OP_DECODE, n_query);
}

}  // namespace msa

extern "C" {

const char* msa_version(void) { return "msa-b200 0.1.0 (sm_100a)"; }

const char* msa_status_string(msa_status st) {
  switch (st) {
    case MSA_OK: return "ok";
    case MSA_ERR_INVALID_ARG: return "invalid argument";
    case MSA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case MSA_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case MSA_ERR_CUDA: return "CUDA error";
    case MSA_ERR_DEVICE: return "device-side error flag set";
    case MSA_ERR_TIMEOUT: return "a bounded device wait ran out";
    default: return "unknown status";
  }
}

size_t msa_workspace_bytes(const msa_params* p, int32_t op, int64_t n_query) {
  Shape s;
  const bool dec = op == MSA_OP_DECODE || op == MSA_OP_DECODE_OFFLOAD;
  if (check_params(p, dec, &s) != MSA_OK) return 0;
  if (dec && n_query < 0) return 0;
  return ws_bytes_for(s, op, n_query);
}

int64_t msa_attn_slab_tokens(const msa_params* p, int32_t op, size_t ws_bytes) {
  Shape s;
  if (check_params(p, false, &s) != MSA_OK) return -1;
  if (op != MSA_OP_SPARSE_ATTN && op != MSA_OP_PREFILL) return -1;
  if (ws_bytes < ws_bytes_for(s, op == MSA_OP_PREFILL ? MSA_OP_PREFILL_MIN : MSA_OP_SPARSE_ATTN_MIN, 0))
    return 0;
  if (!msa::tc_attn_supported(s) || s.seq == 0) return s.seq;
  const size_t fixed = msa::kWsHeader + (op == MSA_OP_PREFILL ? prefill_fixed_ws(s) : 0);
  return msa::tc_attn_slab_tokens(s, ws_bytes - fixed);
}

msa_status msa_pool_keys(const msa_params* p, const void* k, float* kbar, void* kbar_hi,
                         void* kbar_lo, msa_stream_t stream) {
  Shape s;
  msa_status st = check_params(p, false, &s);
  if (st != MSA_OK) return st;
  if (empty_prefill(s)) return MSA_OK;
  if (k == nullptr || kbar == nullptr || !aligned16(k) || !aligned16(kbar))
    return MSA_ERR_INVALID_ARG;
  if ((kbar_hi != nullptr && !aligned16(kbar_hi)) || (kbar_lo != nullptr && !aligned16(kbar_lo)))
    return MSA_ERR_INVALID_ARG;
  if (s.nb > INT32_MAX) return MSA_ERR_UNSUPPORTED;
  return cuda_status(msa::launch_pool_keys(s, k, kbar, kbar_hi, kbar_lo, s.batch,
                                           (cudaStream_t)stream));
}

msa_status msa_block_scores(const msa_params* p, const void* q, const float* kbar, float* scores,
                            msa_stream_t stream) {
  Shape s;
  msa_status st = check_params(p, false, &s);
  if (st != MSA_OK) return st;
  if (empty_prefill(s)) return MSA_OK;
  if (q == nullptr || kbar == nullptr || scores == nullptr) return MSA_ERR_INVALID_ARG;
  if ((double)s.batch * s.hkv * s.seq * s.nb > (double)(((int64_t)1 << 31) - 1) * 256)
    return MSA_ERR_UNSUPPORTED;
  return cuda_status(msa::launch_block_scores(s, q, kbar, scores, (cudaStream_t)stream));
}

msa_status msa_topk_select(const msa_params* p, const void* q, const float* kbar,
                           const void* kbar_hi, const void* kbar_lo, int32_t* idx, void* ws,
                           size_t ws_bytes, msa_stream_t stream) {
  Shape s;
  msa_status st = check_params(p, false, &s);
  if (st != MSA_OK) return st;
  if (empty_prefill(s)) return MSA_OK;
  if (q == nullptr || kbar == nullptr || idx == nullptr || !aligned16(q) || !aligned16(kbar))
    return MSA_ERR_INVALID_ARG;
  if ((kbar_hi != nullptr && !aligned16(kbar_hi)) || (kbar_lo != nullptr && !aligned16(kbar_lo)))
    return MSA_ERR_INVALID_ARG;
  if ((st = check_ws(s, MSA_OP_TOPK_SELECT, 0, ws, ws_bytes)) != MSA_OK) return st;
  return cuda_status(launch_selection(s, q, kbar, kbar_hi, kbar_lo, idx,
                                      reinterpret_cast<uint8_t*>(ws_body(ws)), err_word(ws),
                                      (cudaStream_t)stream));
}

msa_status msa_sparse_attn_fwd(const msa_params* p, const void* q, const void* k, const void* v,
                               const int32_t* idx, void* o, float* lse, void* ws,
                               size_t ws_bytes, msa_stream_t stream) {
  Shape s;
  msa_status st = check_params(p, false, &s);
  if (st != MSA_OK) return st;
  if (empty_prefill(s)) return MSA_OK;
  if (q == nullptr || k == nullptr || v == nullptr || idx == nullptr || o == nullptr)
    return MSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return MSA_ERR_INVALID_ARG;
  if ((st = check_ws(s, MSA_OP_SPARSE_ATTN, 0, ws, ws_bytes)) != MSA_OK) return st;
  return cuda_status(launch_attention(s, q, k, v, idx, o, lse, ws_body(ws),
                                      ws_bytes - msa::kWsHeader, err_word(ws),
                                      (cudaStream_t)stream));
}

msa_status msa_sparse_attn_bwd(const msa_params* p, const void* q, const void* k, const void* v,
                               const void* o, const float* lse, const void* dout,
                               const int32_t* idx, float* dq, float* dk, float* dv, void* ws,
                               size_t ws_bytes, msa_stream_t stream) {
  Shape s;
  msa_status st = check_params(p, false, &s);
  if (st != MSA_OK) return st;
  if (empty_prefill(s)) return MSA_OK;
  if (!msa::tc_attn_bwd_supported(s)) return MSA_ERR_UNSUPPORTED;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || lse == nullptr ||
      dout == nullptr || idx == nullptr || dq == nullptr || dk == nullptr || dv == nullptr)
    return MSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return MSA_ERR_INVALID_ARG;
  if ((st = check_ws(s, MSA_OP_SPARSE_ATTN_BWD, 0, ws, ws_bytes)) != MSA_OK) return st;
  return cuda_status(msa::launch_attn_bwd_tc(s, q, k, v, o, lse, dout, idx, dq, dk, dv,
                                             ws_body(ws), ws_bytes - msa::kWsHeader,
                                             err_word(ws), (cudaStream_t)stream));
}

msa_status msa_prefill_fwd(const msa_params* p, const void* q, const void* k, const void* v,
                           int32_t* idx, void* o, float* lse, void* ws, size_t ws_bytes,
                           msa_stream_t stream) {
  Shape s;
  msa_status st = check_params(p, false, &s);
  if (st != MSA_OK) return st;
  if (empty_prefill(s)) return MSA_OK;
  if (q == nullptr || k == nullptr || v == nullptr || idx == nullptr || o == nullptr)
    return MSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return MSA_ERR_INVALID_ARG;
  if ((st = check_ws(s, MSA_OP_PREFILL, 0, ws, ws_bytes)) != MSA_OK) return st;
  cudaStream_t cs = (cudaStream_t)stream;
  char* body = ws_body(ws);
  float* kbar = reinterpret_cast<float*>(body);
  void* hi = nullptr;
  void* lo = nullptr;
  size_t off = round256(kbar_bytes(s));
  if (kbar_split_bytes(s) > 0) {
    hi = body + off;
    lo = body + off + round256(kbar_split_bytes(s));
    off += 2 * round256(kbar_split_bytes(s));
  }
  uint8_t* flags = reinterpret_cast<uint8_t*>(body + off);
  off += topk_flag_ws(s);
  cudaError_t e = msa::launch_pool_keys(s, k, kbar, hi, lo, s.batch, cs);
  if (e == cudaSuccess) e = launch_selection(s, q, kbar, hi, lo, idx, flags, err_word(ws), cs);
  if (e == cudaSuccess)
    e = launch_attention(s, q, k, v, idx, o, lse, body + off, ws_bytes - msa::kWsHeader - off,
                         err_word(ws), cs);
  return cuda_status(e);
}

msa_status msa_decode_fwd(const msa_params* p, int64_t n_query, const void* q, const float* kbar,
                          const void* kbar_hi, const void* kbar_lo, const void* k_bank,
                          const void* v_bank, int32_t* idx, void* o, float* lse, void* ws,
                          size_t ws_bytes, msa_stream_t stream) {
  Shape s;
  bool tc = false, empty = false;
  msa_status st = msa::check_decode_args(p, n_query, q, kbar, kbar_hi, kbar_lo, k_bank, v_bank,
                                         idx, o, &s, &tc, &empty);
  if (st != MSA_OK || empty) return st;
  if ((st = check_ws(s, MSA_OP_DECODE, n_query, ws, ws_bytes)) != MSA_OK) return st;
  cudaStream_t cs = (cudaStream_t)stream;
  char* sel_ws = ws_body(ws);
  char* att_ws = sel_ws + round256(decode_sel_ws(s, n_query));
  cudaError_t e =
      tc ? msa::launch_topk_decode_tc(s, n_query, q, kbar_hi, kbar_lo, nullptr, idx, sel_ws,
                                      err_word(ws), cs)
         : msa::launch_topk_decode(s, n_query, q, kbar, idx, sel_ws, cs);
  if (e == cudaSuccess)
    e = msa::launch_attn_decode(s, n_query, q, k_bank, v_bank, nullptr, nullptr, idx, o, lse,
                                att_ws, err_word(ws), cs);
  return cuda_status(e);
}

msa_status msa_rope_docwise(const msa_params* p, const int32_t* cu_seqlens, int64_t n_docs,
                            void* q, void* k, double base, msa_stream_t stream) {
  Shape s;
  msa_status st = check_params(p, false, &s);
  if (st != MSA_OK) return st;
  if (n_docs < 1 || !(base > 1.0) || !isfinite(base)) return MSA_ERR_INVALID_ARG;
  if (empty_prefill(s)) return MSA_OK;
  if (n_docs >= INT32_MAX || s.batch * s.seq >= INT32_MAX) return MSA_ERR_UNSUPPORTED;
  if (cu_seqlens == nullptr || q == nullptr || k == nullptr || !aligned16(q) || !aligned16(k))
    return MSA_ERR_INVALID_ARG;
  return cuda_status(msa::launch_rope_docwise(s, cu_seqlens, n_docs, q, k, base,
                                              (cudaStream_t)stream));
}

msa_status msa_prefill_varlen_fwd(const msa_params* p, const int64_t* cu_seqlens, int64_t n_docs,
                                  const void* q, const void* k, const void* v, int32_t* idx,
                                  void* o, float* lse, void* ws, size_t ws_bytes,
                                  msa_stream_t stream) {
  Shape s;
  msa_status st = check_params(p, false, &s);
  if (st != MSA_OK) return st;
  if (p->batch != 1 || n_docs < 1 || cu_seqlens == nullptr) return MSA_ERR_INVALID_ARG;
  if (cu_seqlens[0] != 0 || cu_seqlens[n_docs] != s.seq) return MSA_ERR_INVALID_ARG;
  int64_t longest = 0;
  for (int64_t d = 0; d < n_docs; ++d) {
    const int64_t len = cu_seqlens[d + 1] - cu_seqlens[d];
    if (len < 0) return MSA_ERR_INVALID_ARG;
    if (len > longest) longest = len;
  }
  if (s.seq == 0) return MSA_OK;
  if (q == nullptr || k == nullptr || v == nullptr || idx == nullptr || o == nullptr)
    return MSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return MSA_ERR_INVALID_ARG;
  msa_params one = *p;
  one.seq = longest;
  Shape sl;
  if ((st = check_params(&one, false, &sl)) != MSA_OK) return st;
  if ((st = check_ws(sl, MSA_OP_PREFILL, 0, ws, ws_bytes)) != MSA_OK) return st;
  const size_t es = s.dtype == MSA_BF16 ? 2 : 4;
  for (int64_t d = 0; d < n_docs; ++d) {
    const int64_t a = cu_seqlens[d], len = cu_seqlens[d + 1] - a;
    if (len == 0) continue;
    one.seq = len;
    st = msa_prefill_fwd(&one, (const char*)q + a * s.hq * s.d * es,
                         (const char*)k + a * s.hkv * s.d * es,
                         (const char*)v + a * s.hkv * s.d * es, idx + a * s.hkv * s.topk,
                         (char*)o + a * s.hq * s.d * es, lse ? lse + a * s.hq : nullptr, ws,
                         ws_bytes, stream);
    if (st != MSA_OK) return st;
  }
  return MSA_OK;
}

size_t msa_bank_tiles_bytes(const msa_params* p, int32_t which) {
  Shape s;
  if (check_params(p, true, &s) != MSA_OK) return 0;
  if (which == 0) return msa::bank_kv_tiles_bytes(s);
  if (which == 1) return s.hkv <= msa::kMaxBoundGroups ? msa::bank_kbar_tiles_bytes(s) : 0;
  return 0;
}

// Encoded banks need the tensor-core decode path on both steps.
static bool tiled_decode_supported(const Shape& s) {
  return msa::tc_decode_supported(s) && msa::tc_decode_attn_supported(s);
}

msa_status msa_encode_bank(const msa_params* p, const void* k_bank, const void* v_bank,
                           const void* kbar_hi, const void* kbar_lo, void* k_tiles,
                           void* v_tiles, void* kbar_tiles, msa_stream_t stream) {
  Shape s;
  msa_status st = check_params(p, true, &s);
  if (st != MSA_OK) return st;
  if (s.seq == 0) return MSA_OK;
  if (!tiled_decode_supported(s)) return MSA_ERR_UNSUPPORTED;
  if ((k_tiles != nullptr && k_bank == nullptr) || (v_tiles != nullptr && v_bank == nullptr) ||
      (kbar_tiles != nullptr && (kbar_hi == nullptr || kbar_lo == nullptr)))
    return MSA_ERR_INVALID_ARG;
  if (!aligned16(k_bank) || !aligned16(v_bank) || !aligned16(kbar_hi) || !aligned16(kbar_lo) ||
      !aligned16(k_tiles) || !aligned16(v_tiles) || !aligned16(kbar_tiles))
    return MSA_ERR_INVALID_ARG;
  return cuda_status(msa::launch_encode_bank(s, k_bank, v_bank, kbar_hi, kbar_lo, k_tiles,
                                             v_tiles, kbar_tiles, (cudaStream_t)stream));
}

// Common checks of the encoded-bank decode calls; sets *empty for a call with no work.
static msa_status tiled_checks(const msa_params* p, int64_t n_query, const void* q,
                               const void* const* bufs, int nbufs, const void* ws,
                               size_t ws_bytes, Shape* s, bool* empty) {
  msa_status st = check_params(p, true, s);
  if (st != MSA_OK) return st;
  if (n_query < 0) return MSA_ERR_INVALID_ARG;
  *empty = n_query == 0 || s->seq == 0;
  if (*empty) return MSA_OK;
  if (n_query > 65535 * 64) return MSA_ERR_UNSUPPORTED;
  if (!tiled_decode_supported(*s)) return MSA_ERR_UNSUPPORTED;
  if (q == nullptr || !aligned16(q)) return MSA_ERR_INVALID_ARG;
  for (int i = 0; i < nbufs; ++i)
    if (bufs[i] == nullptr || !aligned16(bufs[i])) return MSA_ERR_INVALID_ARG;
  return check_ws(*s, MSA_OP_DECODE, n_query, ws, ws_bytes);
}

msa_status msa_decode_select_tiled(const msa_params* p, int64_t n_query, const void* q,
                                   const void* kbar_tiles, int32_t* idx, void* ws,
                                   size_t ws_bytes, msa_stream_t stream) {
  Shape s;
  bool empty = false;
  const void* bufs[] = {kbar_tiles, idx};
  msa_status st = tiled_checks(p, n_query, q, bufs, 2, ws, ws_bytes, &s, &empty);
  if (st != MSA_OK || empty) return st;
  return cuda_status(msa::launch_topk_decode_tc(s, n_query, q, nullptr, nullptr, kbar_tiles,
                                                idx, ws_body(ws), err_word(ws),
                                                (cudaStream_t)stream));
}

msa_status msa_decode_attn_tiled(const msa_params* p, int64_t n_query, const void* q,
                                 const void* k_tiles, const void* v_tiles, const int32_t* idx,
                                 void* o, float* lse, void* ws, size_t ws_bytes,
                                 msa_stream_t stream) {
  Shape s;
  bool empty = false;
  const void* bufs[] = {k_tiles, v_tiles, idx, o};
  msa_status st = tiled_checks(p, n_query, q, bufs, 4, ws, ws_bytes, &s, &empty);
  if (st != MSA_OK || empty) return st;
  char* att_ws = ws_body(ws) + round256(decode_sel_ws(s, n_query));
  return cuda_status(msa::launch_attn_decode(s, n_query, q, nullptr, nullptr, k_tiles, v_tiles,
                                             idx, o, lse, att_ws, err_word(ws),
                                             (cudaStream_t)stream));
}

msa_status msa_decode_fwd_tiled(const msa_params* p, int64_t n_query, const void* q,
                                const void* kbar_tiles, const void* k_tiles,
                                const void* v_tiles, int32_t* idx, void* o, float* lse,
                                void* ws, size_t ws_bytes, msa_stream_t stream) {
  msa_status st = msa_decode_select_tiled(p, n_query, q, kbar_tiles, idx, ws, ws_bytes, stream);
  if (st != MSA_OK) return st;
  return msa_decode_attn_tiled(p, n_query, q, k_tiles, v_tiles, idx, o, lse, ws, ws_bytes,
                               stream);
}

msa_status msa_decode_select_shard(const msa_params* p, int64_t n_query, const void* q,
                                   const void* kbar_tiles, int64_t block_offset, uint64_t* keys,
                                   void* ws, size_t ws_bytes, msa_stream_t stream) {
  Shape s;
  bool empty = false;
  const void* bufs[] = {kbar_tiles, keys};
  msa_status st = tiled_checks(p, n_query, q, bufs, 2, ws, ws_bytes, &s, &empty);
  if (st != MSA_OK || empty) return st;
  if (block_offset < 0 || block_offset + s.nb > INT32_MAX / 2) return MSA_ERR_INVALID_ARG;
  return cuda_status(msa::launch_topk_decode_tc(s, n_query, q, nullptr, nullptr, kbar_tiles,
                                                nullptr, ws_body(ws), err_word(ws),
                                                (cudaStream_t)stream, keys, block_offset));
}

msa_status msa_decode_merge_shards(const msa_params* p, int64_t n_query, const uint64_t* keys,
                                   int64_t world, int64_t block_begin, int64_t block_count,
                                   int32_t* idx, int32_t* idx_local, msa_stream_t stream) {
  Shape s;
  msa_status st = check_params(p, true, &s);
  if (st != MSA_OK) return st;
  if (n_query < 0 || world < 1 || block_begin < 0 || block_count < 0 ||
      block_begin + block_count > INT32_MAX / 2)
    return MSA_ERR_INVALID_ARG;
  if (n_query == 0) return MSA_OK;
  if (keys == nullptr || idx == nullptr) return MSA_ERR_INVALID_ARG;
  if (world > 4096 || n_query * s.hkv > ((int64_t)1 << 31)) return MSA_ERR_UNSUPPORTED;
  return cuda_status(msa::launch_merge_shard_keys(keys, world, n_query * s.hkv, (int)s.topk,
                                                  block_begin, block_count, idx, idx_local,
                                                  (cudaStream_t)stream));
}

msa_status msa_decode_combine_shards(const msa_params* p, int64_t n_query, const void* o_parts,
                                     const float* lse_parts, int64_t world, void* o, float* lse,
                                     msa_stream_t stream) {
  Shape s;
  msa_status st = check_params(p, true, &s);
  if (st != MSA_OK) return st;
  if (n_query < 0 || world < 1) return MSA_ERR_INVALID_ARG;
  if (n_query == 0) return MSA_OK;
  if (o_parts == nullptr || lse_parts == nullptr || o == nullptr) return MSA_ERR_INVALID_ARG;
  if (world > 4096 || n_query * s.hq > ((int64_t)1 << 31)) return MSA_ERR_UNSUPPORTED;
  return cuda_status(msa::launch_combine_shards(o_parts, lse_parts, world, n_query * s.hq,
                                                (int)s.d, s.dtype, o, lse,
                                                (cudaStream_t)stream));
}

// Device address under which the GPU reads a host (pinned) or device buffer; null for
// pageable host memory the GPU cannot reach.
static const void* gpu_address(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();                  // clear the error the failed query recorded
    return nullptr;
  }
  if (a.type != cudaMemoryTypeHost && a.type != cudaMemoryTypeDevice) return nullptr;
  return a.devicePointer;
}

msa_status msa_decode_fwd_offload(const msa_params* p, int64_t n_query, const void* q,
                                  const void* kbar_tiles, const void* k_tiles_host,
                                  const void* v_tiles_host, int32_t* idx, void* o, float* lse,
                                  void* ws, size_t ws_bytes, msa_stream_t stream) {
  Shape s;
  msa_status st = check_params(p, true, &s);
  if (st != MSA_OK) return st;
  if (n_query < 0) return MSA_ERR_INVALID_ARG;
  if (n_query == 0 || s.seq == 0) return MSA_OK;
  if (n_query > 65535 * 64) return MSA_ERR_UNSUPPORTED;
  if (!tiled_decode_supported(s) || s.seq % s.block != 0) return MSA_ERR_UNSUPPORTED;
  if (n_query * s.topk * (s.block / 64) > INT32_MAX / 64) return MSA_ERR_UNSUPPORTED;
  if (q == nullptr || kbar_tiles == nullptr || k_tiles_host == nullptr ||
      v_tiles_host == nullptr || idx == nullptr || o == nullptr)
    return MSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kbar_tiles) || !aligned16(k_tiles_host) ||
      !aligned16(v_tiles_host) || !aligned16(o))
    return MSA_ERR_INVALID_ARG;
  if ((st = check_ws(s, MSA_OP_DECODE_OFFLOAD, n_query, ws, ws_bytes)) != MSA_OK) return st;
  const void* kd = gpu_address(k_tiles_host);
  const void* vd = gpu_address(v_tiles_host);
  if (kd == nullptr || vd == nullptr) return MSA_ERR_INVALID_ARG;   // pageable host memory
  cudaStream_t cs = (cudaStream_t)stream;
  char* sel_ws = ws_body(ws);
  char* att_ws = sel_ws + round256(decode_sel_ws(s, n_query));
  char* off_ws = att_ws + round256(msa::decode_attn_ws_bytes(s, n_query));
  cudaError_t e = msa::launch_topk_decode_tc(s, n_query, q, nullptr, nullptr, kbar_tiles, idx,
                                             sel_ws, err_word(ws), cs);
  int32_t* idx_staged = nullptr;
  void *ks = nullptr, *vs = nullptr;
  if (e == cudaSuccess)
    e = msa::launch_offload_stage(s, n_query, idx, kd, vd, kTileBytesKV, off_ws, &idx_staged,
                                  &ks, &vs, cs);
  if (e != cudaSuccess) return MSA_ERR_CUDA;
  // the staging bank: n_query * topk blocks per KV group, addressed by staging slot
  Shape staged = s;
  staged.seq = n_query * s.topk * s.block;
  staged.nb = n_query * s.topk;
  return cuda_status(msa::launch_attn_decode(staged, n_query, q, nullptr, nullptr, ks, vs,
                                             idx_staged, o, lse, att_ws, err_word(ws), cs));
}

msa_status msa_read_device_error(const void* ws, int32_t* bits, msa_stream_t stream) {
  if (ws == nullptr || bits == nullptr) return MSA_ERR_INVALID_ARG;
  int32_t h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, ws, sizeof(int32_t), cudaMemcpyDeviceToHost,
                                  (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return MSA_ERR_CUDA;
  *bits = h;
  return h != 0 ? MSA_ERR_DEVICE : MSA_OK;
}

size_t msa_workspace_size(const msa_params* p, int32_t op, int64_t n_query) {
  return msa_workspace_bytes(p, op, n_query);
}

msa_status msa_get_device_status(const void* ws, msa_stream_t stream) {
  int32_t bits = 0;
  const msa_status st = msa_read_device_error(ws, &bits, stream);
  if (st != MSA_OK && st != MSA_ERR_DEVICE) return st;
  if (bits & MSA_DEVERR_TIMEOUT) return MSA_ERR_TIMEOUT;
  return bits != 0 ? MSA_ERR_DEVICE : MSA_OK;
}

msa_status msa_clear_device_error(void* ws, msa_stream_t stream) {
  if (ws == nullptr) return MSA_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(ws, 0, sizeof(int32_t), (cudaStream_t)stream));
}

}  // extern "C"
