/*
 * msa.h - C ABI of the B200 (sm_100a) block-sparse top-k attention library.
 *
 * The method: pool each KV block into one routing key, score every query against the
 * pooled keys per GQA group, keep the top-k blocks per (query, group), and run exact
 * softmax attention over only the selected K/V blocks.  Sources:
 *   [MiniMax] "MiniMax released MSA: sparse attention speeds up 1M-token context
 *             processing by 28x" (news.hamidun.com), section "How MSA Works": an index
 *             branch picks, for each query and each GQA group, the top-k blocks of keys
 *             and values; a main branch then runs full, exact attention over only those
 *             blocks.  Section "Why Long Context is Hard to Scale": the main branch is
 *             kept exact.
 *   [MoBA]    "MoBA: Mixture of Block Attention for Long-Context LLMs" catalogue card
 *             (ross.abutalabs.com/products/moba.json), field what_it_is: MoE-style
 *             top-k gating over KV blocks; full attention is the case where every block
 *             is selected.
 *   [MSA-DE]  "100 Millionen Token: Gedaechtnis oder Trugbild?" (aitalk.it), section
 *             "Das Gehirn mit zwei Geschwindigkeiten": small routing keys stay on the
 *             GPU and decide relevance; content is attended only once selected; the
 *             routing keys of a memory bank are computed offline.
 * Readings where the pages are silent (they print no formula):
 *   - pooled key = arithmetic mean of the block's keys per KV head (a ragged last block
 *     averages the tokens it holds);
 *   - score(t, g, j) = sum over the group's query heads h of q[t,h] . kbar[j,g]
 *     (unscaled; query head h belongs to group h / (hq/hkv));
 *   - ranking by (score descending, block index ascending);
 *   - causal prefill: the query's own block i = t / block is always selected and the
 *     remaining topk-1 slots go to the best past blocks j < i; inside block i only keys
 *     p <= t are attended; when fewer than topk-1 past blocks exist all are taken;
 *   - decode against a bank: every block is eligible, top `topk`, no mask;
 *   - attention: one softmax per query head over the union of the selected keys,
 *     logits = scale * q . k.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers, row-major and contiguous, 16-byte
 *     aligned.  The caller owns every buffer; the library allocates nothing.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and never synchronise, except msa_read_device_error and
 *     msa_get_device_status.
 *   - Arguments are checked on the host before anything is launched; a failed check
 *     returns MSA_ERR_INVALID_ARG / MSA_ERR_UNSUPPORTED / MSA_ERR_WORKSPACE and launches
 *     nothing.  A launch failure returns MSA_ERR_CUDA.
 *   - Data-dependent faults found on the device (an index out of range, a bounded wait
 *     that ran out) never trap: the kernel skips the offending work and ORs a bit into
 *     the error word at the start of the workspace; read it with msa_read_device_error.
 *   - batch == 0, seq == 0 or n_query == 0 is a valid empty call that launches nothing.
 *   - Results are bitwise deterministic run to run (no floating-point atomics).
 *
 * Layouts (b = batch, S = seq, nb = ceil(S / block), G = hq / hkv):
 *   q    [b, S, hq, d]       k, v [b, S, hkv, d]      o [b, S, hq, d]   (dtype)
 *   kbar [b, nb, hkv, d] fp32; kbar_hi / kbar_lo same shape, bf16 (hi = bf16(kbar),
 *        lo = bf16(kbar - hi))
 *   idx  [b, hkv, S, topk] int32, ascending, padded with -1 at the end
 *   lse  [b, hq, S] fp32, natural log of sum_p exp(scale * q . k_p)
 *   decode: q [n_query, hq, d], bank k/v [S, hkv, d], kbar [nb, hkv, d],
 *           idx [n_query, hkv, topk], o [n_query, hq, d], lse [n_query, hq]
 */
#ifndef MSA_H_
#define MSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MSA_API __attribute__((visibility("default")))
#else
#define MSA_API
#endif

struct CUstream_st;
typedef struct CUstream_st* msa_stream_t; /* same object as cudaStream_t */

typedef enum {
  MSA_OK = 0,
  MSA_ERR_INVALID_ARG = 1, /* null pointer, bad shape, misaligned pointer */
  MSA_ERR_UNSUPPORTED = 2, /* well-formed but outside what the kernels implement */
  MSA_ERR_WORKSPACE = 3,   /* workspace missing, too small or misaligned */
  MSA_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
  MSA_ERR_DEVICE = 5,      /* returned by msa_read_device_error when a bit is set */
  MSA_ERR_TIMEOUT = 6      /* msa_get_device_status: a bounded device wait ran out */
} msa_status;

typedef enum { MSA_F32 = 0, MSA_BF16 = 1 } msa_dtype;

typedef enum {
  MSA_OP_TOPK_SELECT = 0,
  MSA_OP_SPARSE_ATTN = 1,
  MSA_OP_PREFILL = 2,
  MSA_OP_DECODE = 3,
  MSA_OP_SPARSE_ATTN_MIN = 4, /* smallest workspace msa_sparse_attn_fwd accepts */
  MSA_OP_PREFILL_MIN = 5,     /* smallest workspace msa_prefill_fwd accepts */
  MSA_OP_DECODE_OFFLOAD = 6,  /* msa_decode_fwd_offload */
  MSA_OP_SPARSE_ATTN_BWD = 7, /* msa_sparse_attn_bwd, recommended */
  MSA_OP_SPARSE_ATTN_BWD_MIN = 8  /* smallest workspace msa_sparse_attn_bwd accepts */
} msa_op;

/* Device error bits (msa_read_device_error). */
#define MSA_DEVERR_IDX_RANGE 0x1   /* an idx entry outside [-1, nb) or violating causality */
#define MSA_DEVERR_TIMEOUT 0x2     /* a bounded barrier wait ran out */

typedef struct {
  int64_t batch; /* independent sequences (prefill); ignored by decode */
  int64_t seq;   /* tokens per sequence (prefill) or bank tokens (decode) */
  int64_t hq;    /* query heads; hq % hkv == 0 */
  int64_t hkv;   /* key/value heads (GQA groups) */
  int64_t d;     /* head dim: 64 or 128 */
  int64_t block; /* tokens per KV block, >= 1 */
  int64_t topk;  /* selected blocks per (query, group), 1..32, own block included */
  float scale;   /* softmax scale, finite */
  int32_t dtype; /* msa_dtype of q, k, v, o */
} msa_params;

/* Library version string. */
MSA_API const char* msa_version(void);

/* Human-readable name of a status code (static storage). */
MSA_API const char* msa_status_string(msa_status status);

/* Workspace bytes that `op` needs for these shapes (n_query is used by MSA_OP_DECODE
 * only).  Returns 0 when the shapes are invalid.  Pass a buffer of at least this size,
 * 256-byte aligned, to the matching call.  The first 256 bytes hold the device error
 * word; the rest is scratch whose content between calls is unspecified. */
MSA_API size_t msa_workspace_bytes(const msa_params* p, int32_t op, int64_t n_query);

/* Tokens per slab that msa_sparse_attn_fwd (op MSA_OP_SPARSE_ATTN) or msa_prefill_fwd
 * (op MSA_OP_PREFILL) processes at a time when given ws_bytes of workspace: p->seq for one
 * pass, 0 when ws_bytes is below the minimum, -1 for invalid params or op.  Each slab
 * is one more round of the attention's six kernel launches.  Host-only. */
MSA_API int64_t msa_attn_slab_tokens(const msa_params* p, int32_t op, size_t ws_bytes);

/* Step 1, block pooling ([MSA-DE] routing keys; [MoBA] KV blocks):
 *   kbar[b,j,g,:] = (1/n_j) * sum_{t in block j} k[b,t,g,:],  n_j = tokens in block j.
 * kbar (fp32) is required; kbar_hi / kbar_lo (bf16 split planes) may each be NULL.
 * Accumulates in fp32 in token order.  Applied to a memory bank this is the offline
 * encoding of its routing keys. */
MSA_API msa_status msa_pool_keys(const msa_params* p, const void* k, float* kbar, void* kbar_hi,
                         void* kbar_lo, msa_stream_t stream);

/* Step 2 materialised, for inspection and small shapes ([MiniMax] index branch):
 *   scores[b,g,t,j] = sum_{h in group g} q[b,t,h,:] . kbar[b,j,g,:]   for j < t/block,
 *   -inf for j >= t/block.  fp32, [b, hkv, S, nb].  The fused selection never stores
 *   scores; this entry is O(S * nb) memory. */
MSA_API msa_status msa_block_scores(const msa_params* p, const void* q, const float* kbar,
                            float* scores, msa_stream_t stream);

/* Steps 2+3 fused, causal prefill ([MiniMax] index branch; [MoBA] top-k gating):
 * idx[b,g,t,:] = {t/block} U top-(topk-1) past blocks by (score desc, index asc),
 * ascending, -1 padded.  kbar is required; kbar_hi / kbar_lo may be NULL (they are
 * used when present).  ws: msa_workspace_bytes(p, MSA_OP_TOPK_SELECT, 0). */
MSA_API msa_status msa_topk_select(const msa_params* p, const void* q, const float* kbar,
                           const void* kbar_hi, const void* kbar_lo, int32_t* idx, void* ws,
                           size_t ws_bytes, msa_stream_t stream);

/* Step 4, causal prefill ([MiniMax] main branch, exact):
 *   o[b,t,h,:] = sum_{p in U} softmax_p(scale * q[b,t,h,:] . k[b,p,g,:]) v[b,p,g,:],
 *   U = keys of the blocks in idx[b,g,t,:] (entries -1 skipped), keeping p <= t.
 * lse may be NULL.  Entries outside [-1, nb) or after the own block set
 * MSA_DEVERR_IDX_RANGE and are skipped.  ws: msa_workspace_bytes(p, MSA_OP_SPARSE_ATTN) is
 * the recommended size (the whole sequence in one pass, or token slabs of about 32 GiB of
 * partials); any size from msa_workspace_bytes(p, MSA_OP_SPARSE_ATTN_MIN) up is accepted,
 * and the bf16 d = 128 path then processes the sequence in token slabs (multiples of 2048
 * tokens) that fit ws_bytes: same results, more launches. */
MSA_API msa_status msa_sparse_attn_fwd(const msa_params* p, const void* q, const void* k, const void* v,
                               const int32_t* idx, void* o, float* lse, void* ws,
                               size_t ws_bytes, msa_stream_t stream);

/* Backward of step 4 ([MSA-DE] "Eleganter Proof-of-Concept oder fertiges System?": the
 * router and the sparse attention are trained end to end).  The selection idx is held
 * fixed (top-k passes no gradient, so the pooled keys get none through it); the rest is
 * the exact gradient of the attention over each row's selected keys:
 *   P_p = exp(scale q.k_p - lse), D = dO . o (per row and head),
 *   dv_p += P_p dO,  dk_p += scale P_p (dO.v_p - D) q,  dq = scale sum_p P_p (dO.v_p - D) k_p,
 * summed over every (row, head) that attends key p.  Inputs as for msa_sparse_attn_fwd plus
 * its outputs o [b,S,hq,d] and lse [b,hq,S] (required) and the upstream gradient dout
 * [b,S,hq,d]; outputs dq [b,S,hq,d], dk, dv [b,S,hkv,d], all fp32, overwritten.
 * Supported: bf16, d = 128, block a multiple of 128, G in {1,2,4,8}, topk * block/128 <= 64
 * (else MSA_ERR_UNSUPPORTED).  ws: msa_workspace_bytes(p, MSA_OP_SPARSE_ATTN_BWD, 0)
 * recommended, at least MSA_OP_SPARSE_ATTN_BWD_MIN (token slabs of 2048 multiples).
 * Bitwise deterministic: every sum runs in a fixed order. */
MSA_API msa_status msa_sparse_attn_bwd(const msa_params* p, const void* q, const void* k,
                                       const void* v, const void* o, const float* lse,
                                       const void* dout, const int32_t* idx, float* dq,
                                       float* dk, float* dv, void* ws, size_t ws_bytes,
                                       msa_stream_t stream);

/* Whole causal prefill: msa_pool_keys -> msa_topk_select -> msa_sparse_attn_fwd, with the
 * pooled keys kept in the workspace.  idx is written (caller-owned, [b,hkv,S,topk]);
 * lse may be NULL.  ws: msa_workspace_bytes(p, MSA_OP_PREFILL, 0) recommended, at least
 * msa_workspace_bytes(p, MSA_OP_PREFILL_MIN, 0) (slabbed attention, as above). */
MSA_API msa_status msa_prefill_fwd(const msa_params* p, const void* q, const void* k, const void* v,
                           int32_t* idx, void* o, float* lse, void* ws, size_t ws_bytes,
                           msa_stream_t stream);

/* Document-wise rotary positions ([MSA-DE] "Das Gehirn mit zwei Geschwindigkeiten": the
 * position counter restarts at zero at the start of every document), applied in place:
 * for the T = p->batch * p->seq packed tokens of q [T, hq, d] and k [T, hkv, d], dimensions
 * i and i + d/2 of every head are rotated by pos * base^(-2i/d):
 *   (x_i, x_{i+d/2}) -> (x_i cos a - x_{i+d/2} sin a, x_{i+d/2} cos a + x_i sin a),
 * pos = t - cu_seqlens[doc(t)].  cu_seqlens: DEVICE int32 array of the n_docs + 1 document
 * boundaries, 0 = cu_seqlens[0] <= ... <= cu_seqlens[n_docs] = T (other contents give
 * meaningless positions but no out-of-range access).  base > 1.  Angles are formed in
 * fp64, the rotation in fp32, the result rounded to the tensors' dtype.  Values are not
 * rotated.  The rotated q and k then feed every other call unchanged. */
MSA_API msa_status msa_rope_docwise(const msa_params* p, const int32_t* cu_seqlens,
                                    int64_t n_docs, void* q, void* k, double base,
                                    msa_stream_t stream);

/* Causal prefill of packed documents, each its own sequence ([MSA-DE] "Das Gehirn mit
 * zwei Geschwindigkeiten": documents are processed one by one): p->batch must be 1 and
 * p->seq = T, the packed token count; cu_seqlens is a HOST int64 array of the n_docs + 1
 * boundaries (0 first, T last, nondecreasing; else MSA_ERR_INVALID_ARG).  Document d =
 * tokens [a, b) with a = cu_seqlens[d], b = cu_seqlens[d+1]: its blocks start at a, no
 * selection or attention crosses a boundary, and the results are those of
 * msa_prefill_fwd on that document alone, laid out as:
 *   q, o [T, hq, d]; k, v [T, hkv, d]   (packed, natural layout);
 *   idx: document d's [hkv, b-a, topk] at element offset a * hkv * topk, block ids
 *        counted from the document's first block;
 *   lse (may be NULL): document d's [hq, b-a] at element offset a * hq.
 * ws: at least msa_workspace_bytes(p', MSA_OP_PREFILL_MIN, 0) where p' is p with seq =
 * the longest document (MSA_OP_PREFILL recommended).  The documents run one after the
 * other on `stream` (one msa_prefill_fwd each: about 9 launches per document, so many
 * short documents are bound by launch cost). */
MSA_API msa_status msa_prefill_varlen_fwd(const msa_params* p, const int64_t* cu_seqlens,
                                          int64_t n_docs, const void* q, const void* k,
                                          const void* v, int32_t* idx, void* o, float* lse,
                                          void* ws, size_t ws_bytes, msa_stream_t stream);

/* Decode against a memory bank ([MSA-DE] routing keys in GPU memory decide which content
 * is attended; [MiniMax] per query and GQA group top-k):  for each query n and group g,
 * idx[n,g,:] = top-`topk` of all nb bank blocks by (score desc, index asc), ascending;
 * then exact attention of the group's heads over those blocks' keys, no mask.
 * p->seq is the number of bank tokens, p->batch is ignored.  The bank's pooled keys come
 * from msa_pool_keys, computed once when the bank is written ([MSA-DE]: offline):
 *   - kbar_hi and kbar_lo (bf16 split planes, [nb, hkv, d]) both given, with bf16 queries
 *     and d = 128: the tensor-core scan reads only the planes and kbar may be NULL;
 *   - otherwise kbar (fp32) is required and the fp32 SIMT scan runs.
 * ws: msa_workspace_bytes(p, MSA_OP_DECODE, n_query) (covers both scans). */
MSA_API msa_status msa_decode_fwd(const msa_params* p, int64_t n_query, const void* q,
                                  const float* kbar, const void* kbar_hi, const void* kbar_lo,
                                  const void* k_bank, const void* v_bank, int32_t* idx, void* o,
                                  float* lse, void* ws, size_t ws_bytes, msa_stream_t stream);

/* Encoded decode bank ([MSA-DE]: the bank and its routing keys are prepared offline, when
 * the bank is written).  Same method and results as msa_decode_fwd; only the memory
 * layout of the bank differs, chosen so that each selected tile is one contiguous run:
 *   k_tiles, v_tiles  [hkv][ceil(S/64)][2][64][64] bf16: per KV head, 64-key tiles, each
 *                     as two 64-dim halves of 64 rows x 128 bytes; inside a half, the
 *                     16-byte chunk c of row r is stored at chunk position c ^ (r % 8);
 *                     rows past S are zero.  msa_bank_tiles_bytes(p, 0) bytes each.
 *   kbar_tiles        [2][hkv][ceil(nb/128)][2][128][64] bf16: the hi planes, then the lo
 *                     planes of the pooled keys, per KV head in 128-block chunks, the
 *                     same half/row/chunk order and swizzle; rows past nb are zero.  Then
 *                     256 bytes: fp32 [2][hkv] = max over blocks of ||lo_j||_2, then of
 *                     ||hi_j||_2, per KV head (the selection's error bound, below).
 *                     msa_bank_tiles_bytes(p, 1) bytes.
 * Supported: bf16, d = 128, block a multiple of 64, G in {1, 2, 4, 8}, hkv <= 32 (else
 * MSA_ERR_UNSUPPORTED).  msa_bank_tiles_bytes returns 0 for invalid shapes or `which`,
 * and for which = 1 when hkv > 32.
 * On large encoded banks (at least 1017 chunks of 128 blocks per KV head, about 8.3M
 * tokens at block 64) the selection reads the lo plane only where it matters: a scan of
 * the hi plane proposes each row's 64 best blocks, these are scored exactly, and a row is
 * accepted when the bound max||lo|| * ||q|| on the dropped term proves that no other
 * block can reach its top k; if any row is not proven (near-equal scores across many
 * blocks, such as exact ties), the whole bank is scanned exactly as well.  Smaller banks
 * scan both planes.  The selection is the natural-layout one in every case. */
MSA_API size_t msa_bank_tiles_bytes(const msa_params* p, int32_t which);

/* Writes the encoded images of a bank in the natural layout (k_bank, v_bank [S, hkv, d];
 * kbar_hi, kbar_lo [nb, hkv, d] from msa_pool_keys).  Any of k_tiles, v_tiles,
 * kbar_tiles may be NULL (that image is skipped); the matching inputs are then unused. */
MSA_API msa_status msa_encode_bank(const msa_params* p, const void* k_bank, const void* v_bank,
                                   const void* kbar_hi, const void* kbar_lo, void* k_tiles,
                                   void* v_tiles, void* kbar_tiles, msa_stream_t stream);

/* The two steps of a decode over an encoded bank, for callers that schedule them apart
 * (msa_decode_fwd_tiled below is the two in sequence).  Both take the same decode
 * workspace; the selection writes idx [n_query, hkv, topk] as msa_decode_fwd does, the
 * attention reads it (entries -1 skipped, others must be in [0, nb): an out-of-range
 * entry is skipped and sets MSA_DEVERR_IDX_RANGE). */
MSA_API msa_status msa_decode_select_tiled(const msa_params* p, int64_t n_query, const void* q,
                                           const void* kbar_tiles, int32_t* idx, void* ws,
                                           size_t ws_bytes, msa_stream_t stream);
MSA_API msa_status msa_decode_attn_tiled(const msa_params* p, int64_t n_query, const void* q,
                                         const void* k_tiles, const void* v_tiles,
                                         const int32_t* idx, void* o, float* lse, void* ws,
                                         size_t ws_bytes, msa_stream_t stream);

/* msa_decode_fwd over an encoded bank: the same selection (tensor-core scan of the
 * pooled-key planes) and the same attention, fed by 1-D bulk copies.
 * ws: msa_workspace_bytes(p, MSA_OP_DECODE, n_query). */
MSA_API msa_status msa_decode_fwd_tiled(const msa_params* p, int64_t n_query, const void* q,
                                        const void* kbar_tiles, const void* k_tiles,
                                        const void* v_tiles, int32_t* idx, void* o, float* lse,
                                        void* ws, size_t ws_bytes, msa_stream_t stream);

/* Memory Parallel decode ([MSA-DE] "Das Gehirn mit zwei Geschwindigkeiten": each GPU
 * holds part of the routing keys, the queries are broadcast to all, the relevance scores
 * are aggregated, and only the selected content is loaded).  The bank's blocks are split
 * into contiguous ranges, one per rank; every shard but the last holds a whole number of
 * blocks.  One decode step on every rank:
 *   1. msa_decode_select_shard over the rank's shard (its own encoded planes, p->seq = the
 *      shard's tokens): the shard's best topk 64-bit keys per (query, group),
 *      keys [n_query, hkv, topk], sorted descending; a key holds the score's
 *      order-preserving bits above the complement of the bank-wide block id
 *      (block_offset = the shard's first block), 0 = empty.  Workspace as for
 *      msa_decode_select_tiled.
 *   2. the caller all-gathers the keys of all ranks into [world, n_query, hkv, topk]
 *      (rank order) and calls msa_decode_merge_shards: idx [n_query, hkv, topk] gets the
 *      bank-wide selection (ascending, -1 padded) - exactly the unsharded top-k, since each
 *      block of the bank-wide top-k is in its own shard's top-k - and idx_local (nullable)
 *      the ids, local to the shard [block_begin, block_begin + block_count), of the
 *      selected blocks this rank owns, -1 elsewhere.
 *   3. msa_decode_attn_tiled over the rank's shard with idx_local: the rank's partial o and
 *      lse (o = 0 and lse = -inf for a row with no owned block).
 *   4. the caller all-gathers o [world, n_query, hq, d] (dtype) and lse
 *      [world, n_query, hq] and calls msa_decode_combine_shards: o, lse = the softmax over
 *      the whole selection (partials weighted by exp(lse_r - max), in rank order).
 * The three calls are asynchronous on `stream`, allocate nothing and check their arguments
 * on the host first (p->topk, p->hkv, p->hq and p->d give the shapes; p->seq is unused by
 * steps 2 and 4). */
MSA_API msa_status msa_decode_select_shard(const msa_params* p, int64_t n_query, const void* q,
                                           const void* kbar_tiles, int64_t block_offset,
                                           uint64_t* keys, void* ws, size_t ws_bytes,
                                           msa_stream_t stream);
MSA_API msa_status msa_decode_merge_shards(const msa_params* p, int64_t n_query,
                                           const uint64_t* keys, int64_t world,
                                           int64_t block_begin, int64_t block_count,
                                           int32_t* idx, int32_t* idx_local,
                                           msa_stream_t stream);
MSA_API msa_status msa_decode_combine_shards(const msa_params* p, int64_t n_query,
                                             const void* o_parts, const float* lse_parts,
                                             int64_t world, void* o, float* lse,
                                             msa_stream_t stream);

/* Decode against a bank whose content stays in host memory ([MSA-DE] "Das Gehirn mit
 * zwei Geschwindigkeiten": the routing keys stay in GPU memory, the content keys and
 * values are moved to the CPU's system RAM and brought to the GPU only once the router
 * selects them; "100 Millionen Token auf 2xA800: Zu welchem Preis?" puts that transfer on
 * PCIe).  Same method, arguments and results as msa_decode_fwd_tiled, except:
 *   - k_tiles_host / v_tiles_host: the encoded K/V images (msa_encode_bank layout) in
 *     PINNED host memory (cudaHostAlloc / cudaHostRegister, or a pinned torch tensor), which
 *     the GPU reads directly (unified addressing); pageable memory is rejected
 *     (MSA_ERR_INVALID_ARG).  Device memory is accepted as well.  kbar_tiles is in HBM.
 *   - after the selection, each selected (KV group, block) is fetched once, however many
 *     queries selected it, into an HBM staging bank in the workspace; the attention then
 *     runs on the staged copy, so o, lse and idx are bitwise msa_decode_fwd_tiled's.
 *   - p->seq must be a multiple of p->block (else MSA_ERR_UNSUPPORTED).
 * ws: msa_workspace_bytes(p, MSA_OP_DECODE_OFFLOAD, n_query): the decode workspace plus the
 * staging bank (n_query x topk x block keys of K and V per KV group: 512 MiB for 64
 * queries, 8 groups, top-32 blocks of 64) and per-block marks (5 bytes per bank block and
 * group). */
MSA_API msa_status msa_decode_fwd_offload(const msa_params* p, int64_t n_query, const void* q,
                                          const void* kbar_tiles, const void* k_tiles_host,
                                          const void* v_tiles_host, int32_t* idx, void* o,
                                          float* lse, void* ws, size_t ws_bytes,
                                          msa_stream_t stream);

/* Bytes of the fixed device scratch used by msa_decode_fwd_static (32 MiB). */
#define MSA_DECODE_STATIC_SCRATCH_BYTES ((size_t)32 << 20)

/* Decode without a caller workspace, for callers that cannot allocate device memory
 * where they run a decode step (for example a runtime that reserves all device memory up
 * front and forbids allocation on its hot path, or a plug-in whose host framework owns
 * every allocation and passes only the step's tensors).  The pages have no counterpart:
 * this is a deployment variant of msa_decode_fwd, with the same arguments minus the
 * workspace, the same kernels and the same results.
 *   - Scratch: a file-scope device array of MSA_DECODE_STATIC_SCRATCH_BYTES that every
 *     GPU loading this library keeps until the process exits.  The call allocates
 *     nothing (no cudaMalloc/cudaFree, no allocating library routine).
 *   - Checks: every argument is checked first, with msa_decode_fwd's statuses, before
 *     any CUDA call.  Returns MSA_ERR_WORKSPACE, launching nothing, when
 *     msa_workspace_bytes(p, MSA_OP_DECODE, n_query) exceeds the array (64 queries x 32
 *     heads against a 10M-token bank need about 28 MB).
 *   - Set-up: the first call on a device looks up the array's device address with that
 *     device current (cudaGetSymbolAddress) and caches it for the process; make that
 *     first call before any stream capture.  cudaDeviceReset on a device invalidates the
 *     cached address: do not call this entry on that device again in the same process.
 *   - Sharing: every call on a device uses the same array, which keeps the last call's
 *     contents; the call clears what must start at zero.  Calls that overlap on the GPU
 *     (concurrent streams, or several host threads) race on the array: serialise them.
 *   - Device error bits: the call returns MSA_OK even when a kernel skipped work (a
 *     bounded wait ran out, an index out of range); msa_decode_static_read_error reads
 *     the bits of the last call on the current device. */
MSA_API msa_status msa_decode_fwd_static(const msa_params* p, int64_t n_query, const void* q,
                                         const float* kbar, const void* kbar_hi,
                                         const void* kbar_lo, const void* k_bank,
                                         const void* v_bank, int32_t* idx, void* o, float* lse,
                                         msa_stream_t stream);

/* The device error word of msa_decode_fwd_static's array on the current device (the last
 * call's bits: each call clears them first), read after synchronising `stream`; returns
 * MSA_ERR_DEVICE when any bit is set, else MSA_OK, and MSA_ERR_INVALID_ARG for a null
 * `bits`.  No other call may be using the array meanwhile. */
MSA_API msa_status msa_decode_static_read_error(int32_t* bits, msa_stream_t stream);

/* Copies the workspace's device error word to *bits after synchronising `stream`;
 * returns MSA_ERR_DEVICE when any bit is set, else MSA_OK. */
MSA_API msa_status msa_read_device_error(const void* ws, int32_t* bits, msa_stream_t stream);

/* Clears the workspace's device error word (asynchronous on `stream`). */
MSA_API msa_status msa_clear_device_error(void* ws, msa_stream_t stream);

/* The same two queries under the names of the library's original interface sketch:
 * msa_workspace_size is msa_workspace_bytes; msa_get_device_status synchronises `stream`
 * and returns MSA_ERR_TIMEOUT when the workspace's error word holds MSA_DEVERR_TIMEOUT,
 * MSA_ERR_DEVICE when it holds any other bit, else MSA_OK (the word is left as it is). */
MSA_API size_t msa_workspace_size(const msa_params* p, int32_t op, int64_t n_query);
MSA_API msa_status msa_get_device_status(const void* ws, msa_stream_t stream);

/* Diagnostic: y[i] = the attention softmax's own base-2 exponential of x[i] (device
 * fp32 arrays of n elements), the FMA-pipe cubic that takes part of the softmax's
 * exponentials off the MUFU unit.  [MiniMax] "How MSA Works" keeps the main branch exact;
 * this entry lets a caller hold that helper to its bound: relative error <= 7.5e-5 for
 * x >= -125.5, a value in [0, 2^-125] below.  The pages have no counterpart.
 * Asynchronous on `stream`. */
MSA_API msa_status msa_exp2_poly_eval(const float* x, float* y, int64_t n, msa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H_ */
