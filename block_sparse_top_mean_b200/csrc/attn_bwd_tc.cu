// Backward pass of step 4 on the tensor cores (bf16, d = 128).
//
// "100 Millionen Token: Gedaechtnis oder Trugbild?" (aitalk.it), section "Eleganter
// Proof-of-Concept oder fertiges System?": the router and the sparse attention are
// trained end to end.  The selection is piecewise constant and passes no gradient; the
// rest is the gradient of exact softmax attention over each row's selected keys:
//   P = softmax(scale q.k) (recomputed from the forward's lse), dP = dO . v,
//   dS = P (dP - D) with D = dO . O per row,
//   dV_p += P_p dO,  dK_p += scale dS_p q,  dQ = scale sum_p dS_p k_p.
//
// Key-centric, like the forward: the selection is inverted into per-(sequence, group,
// block, 128-key segment) lists of (token, slot) entries, and one tile = the G heads of
// 128/G such tokens (128 rows) against the segment's 128 keys.  A CTA owns whole segments
// (dealt out by tile count, bwd_balance_kernel), so dK and dV of a key accumulate in TMEM
// over all tiles that read it, in the order of the segment's entries, and are written
// once.  That order is fixed: the fill places entries in a sequence that depends only on
// idx (one warp per 2048-token range walks its tokens in order), so results are bitwise
// reproducible.  Per tile:
//   S = Q K^T, dP = dO V^T        tcgen05, both operands K-major in shared memory
//   P, dS (bf16, scale folded into dS) written to shared memory by the 128 row threads
//   dV += P^T dO, dK += dS^T Q   tcgen05, A = P^T / dS^T read MN-major from the same tiles
//   dQ_part = dS K                tcgen05 into S's TMEM columns, written as a bf16 partial
// TMEM: S (and then dQ) [0,128), dP [128,256), dV [256,384), dK [384,512); lanes = rows
// for S/dP/dQ and = keys for dV/dK.  dQ partials are merged per row in slot order by
// bwd_merge_dq_kernel; dK and dV accumulate in fp32 across token slabs (one slab after
// the other, each key in exactly one segment, so no two CTAs touch the same key).
#include <cudaTypedefs.h>
#include <math_constants.h>

#include "common.cuh"
#include "fastmath.cuh"
#include "sm100.cuh"

namespace msa {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kRowsT = 128;               // rows per tile
constexpr int kSeg = 128;                 // keys per segment (one MMA N / K extent)
constexpr uint32_t kHalf = 16384;         // 128 rows x 128 B: one 64-column half
constexpr uint32_t kTile = 2 * kHalf;     // a 128 x 128 bf16 operand tile
constexpr int kTokRange = 2048;           // tokens per inversion CTA
constexpr float kLog2e = 1.4426950408889634f;

struct BGeom {
  int64_t S, nb, block, nseg;
  int64_t t_base, t_end, slab;
  int hq, hkv, G, topk, nsub, kslots, tpt, n_ranges;
  float scale, scale_log2;
};

// Segment sub of block j holds keys [j*block + sub*128, +128); whether token t (own block
// `own`) reads any of them.
__device__ __forceinline__ bool seg_has_keys(int j, int own, int t, int sub, const BGeom& g) {
  const int64_t lo = (int64_t)j * g.block + (int64_t)sub * kSeg;
  if ((int64_t)sub * kSeg >= g.block || lo >= g.S) return false;
  return j < own || lo <= t;
}

// ------------------------------------------------------------------ deterministic inversion
// counts[bg][range][seg]: entries of each segment from each 2048-token range.
__global__ void __launch_bounds__(512)
bwd_count_kernel(const int32_t* __restrict__ idx, int* __restrict__ counts, int* err, BGeom g) {
  extern __shared__ int hist[];
  const int nbs = (int)g.nb * g.nsub;
  const int range = blockIdx.x, bg = blockIdx.y;
  const int t0 = (int)g.t_base + range * kTokRange;
  const int t1 = (int)min((int64_t)t0 + kTokRange, g.t_end);
  for (int i = threadIdx.x; i < nbs; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int32_t* irow = idx + ((int64_t)bg * g.S + t0) * g.topk;
  const int n = (t1 - t0) * g.topk;
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const int j = irow[e];
    if (j == -1) continue;
    const int t = t0 + e / g.topk;
    const int own = t / (int)g.block;
    if (j < -1 || j >= g.nb || j > own) {
      set_device_error(err, MSA_DEVERR_IDX_RANGE);
      continue;
    }
    for (int sub = 0; sub < g.nsub; ++sub)
      if (seg_has_keys(j, own, t, sub, g)) atomicAdd(&hist[j * g.nsub + sub], 1);
  }
  __syncthreads();
  int* row = counts + ((int64_t)bg * g.n_ranges + range) * nbs;
  for (int i = threadIdx.x; i < nbs; i += blockDim.x) row[i] = hist[i];
}

// Per segment: exclusive prefix over the ranges (in place) and the segment's total.
__global__ void bwd_colscan_kernel(int* __restrict__ counts, int* __restrict__ totals, BGeom g) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t nbs = g.nb * g.nsub;
  if (i >= (int64_t)(g.nseg)) return;
  const int64_t bg = i / nbs, s = i % nbs;
  int* col = counts + bg * g.n_ranges * nbs + s;
  int run = 0;
  for (int r = 0; r < g.n_ranges; ++r) {
    const int c = col[(int64_t)r * nbs];
    col[(int64_t)r * nbs] = run;
    run += c;
  }
  totals[i] = run;
}

// Single-CTA exclusive scans: seg_off (entries) and tile_off (tiles of tpt entries).
__global__ void __launch_bounds__(1024)
bwd_scan_kernel(const int* __restrict__ totals, int* __restrict__ seg_off,
                int* __restrict__ tile_off, int* __restrict__ n_tiles, int64_t nseg, int tpt) {
  __shared__ long long s_e[1024], s_t[1024];
  const int tid = threadIdx.x;
  const int64_t per = (nseg + 1023) / 1024;
  const int64_t lo = tid * per, hi = lo + per < nseg ? lo + per : nseg;
  long long se = 0, st = 0;
  for (int64_t i = lo; i < hi; ++i) { se += totals[i]; st += (totals[i] + tpt - 1) / tpt; }
  s_e[tid] = se; s_t[tid] = st;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    long long a = tid >= off ? s_e[tid - off] : 0, b = tid >= off ? s_t[tid - off] : 0;
    __syncthreads();
    s_e[tid] += a; s_t[tid] += b;
    __syncthreads();
  }
  long long ce = s_e[tid] - se, ct = s_t[tid] - st;
  for (int64_t i = lo; i < hi; ++i) {
    seg_off[i] = (int)ce; tile_off[i] = (int)ct;
    ce += totals[i]; ct += (totals[i] + tpt - 1) / tpt;
  }
  if (tid == 1023) { seg_off[nseg] = (int)s_e[1023]; tile_off[nseg] = (int)s_t[1023];
                     *n_tiles = (int)s_t[1023]; }
}

// One warp per (bg, token range): walks the range's tokens 32 at a time (lane = token)
// and, for each slot and segment part in order, places the entries of equal segments by
// lane order after the range's earlier entries: a sequence fixed by idx alone.
__global__ void __launch_bounds__(32)
bwd_fill_kernel(const int32_t* __restrict__ idx, const int* __restrict__ base,
                const int* __restrict__ seg_off, int* __restrict__ entries, BGeom g) {
  extern __shared__ int run[];                        // entries placed so far per segment
  const int nbs = (int)g.nb * g.nsub;
  const int range = blockIdx.x, bg = blockIdx.y, lane = threadIdx.x;
  for (int i = lane; i < nbs; i += 32) run[i] = 0;
  __syncwarp();
  const int t0 = (int)g.t_base + range * kTokRange;
  const int t1 = (int)min((int64_t)t0 + kTokRange, g.t_end);
  const int* bs = base + ((int64_t)bg * g.n_ranges + range) * nbs;
  const int* so = seg_off + (int64_t)bg * nbs;
  for (int tr = t0; tr < t1; tr += 32) {
    const int t = tr + lane;
    const bool live = t < t1;
    const int own = t / (int)g.block;
    for (int slot = 0; slot < g.topk; ++slot) {
      const int j = live ? idx[((int64_t)bg * g.S + t) * g.topk + slot] : -1;
      const bool ok_j = j >= 0 && j < g.nb && j <= own;
      for (int sub = 0; sub < g.nsub; ++sub) {
        const bool has = ok_j && seg_has_keys(j, own, t, sub, g);
        const int seg = has ? j * g.nsub + sub : -1 - lane;   // unique non-matches
        const unsigned peers = __match_any_sync(0xffffffffu, seg);
        if (has) {
          const int rank = __popc(peers & ((1u << lane) - 1u));
          const int pos = so[seg] + bs[seg] + run[seg] + rank;
          entries[pos] = (t << 6) | (slot * g.nsub + sub);
        }
        __syncwarp();
        if (has && __ffs(peers) - 1 == lane) run[seg] += __popc(peers);
        __syncwarp();
      }
    }
  }
}

// tiles[tile] = (segment, first entry, entries, sequence * hkv + group)
__global__ void bwd_tile_table_kernel(const int* __restrict__ totals, const int* __restrict__ seg_off,
                                      const int* __restrict__ tile_off,
                                      const int* __restrict__ n_tiles, int4* __restrict__ tiles,
                                      int64_t nseg, int tpt, int64_t nseg_per_bg) {
  const int64_t tile = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (tile >= *n_tiles) return;
  int64_t lo = 0, hi = nseg;                       // largest s with tile_off[s] <= tile
  while (hi - lo > 1) {
    const int64_t mid = (lo + hi) / 2;
    if (tile_off[mid] <= tile) lo = mid; else hi = mid;
  }
  while (lo + 1 < nseg && tile_off[lo + 1] <= tile) ++lo;
  const int k = (int)(tile - tile_off[lo]);
  const int cnt = min(tpt, totals[lo] - k * tpt);
  tiles[tile] = make_int4((int)lo, seg_off[lo] + k * tpt, cnt, (int)(lo / nseg_per_bg));
}

// The CTAs' segment lists: every non-empty segment goes to exactly one CTA, which runs
// all of its tiles (dK and dV of its keys accumulate in that CTA's TMEM).  Segments of at
// least a quarter of a CTA's fair share of tiles are dealt out first, round-robin; the
// others fill each CTA up to the fair share in segment order.  Without such segments the
// plain round-robin over all segments is kept (seg_beg[kMaxBwdCtas] = 1), which measured
// faster when every segment is small.  The assignment changes neither any result nor its
// bits: a segment's tiles run in entry order wherever it runs.
constexpr int kBalThreads = 1024;
constexpr int kMaxBwdCtas = 1024;
__global__ void __launch_bounds__(kBalThreads)
bwd_balance_kernel(const int* __restrict__ tile_off, int64_t nseg, int ncta,
                   int* __restrict__ seg_list, int* __restrict__ seg_beg) {
  __shared__ long long s_a[kBalThreads], s_b[kBalThreads];
  __shared__ long long cap_off[kMaxBwdCtas + 1];
  __shared__ int load[kMaxBwdCtas], cnt[kMaxBwdCtas], fill[kMaxBwdCtas];
  const int tid = threadIdx.x;
  const long long total = tile_off[nseg];
  const long long fair = (total + ncta - 1) / ncta;
  const long long big = fair / 4 > 1 ? fair / 4 : 1;
  for (int c = tid; c < ncta; c += kBalThreads) { load[c] = 0; cnt[c] = 0; fill[c] = 0; }
  // per-thread contiguous ranges of segments: ranks of big segments, small-tile prefixes
  const int64_t per = (nseg + kBalThreads - 1) / kBalThreads;
  const int64_t lo = tid * per, hi = lo + per < nseg ? lo + per : nseg;
  long long nbig = 0, small = 0;
  for (int64_t i = lo; i < hi; ++i) {
    const long long t = tile_off[i + 1] - tile_off[i];
    if (t >= big) ++nbig; else small += t;
  }
  s_a[tid] = nbig;
  s_b[tid] = small;
  __syncthreads();
  for (int off = 1; off < kBalThreads; off <<= 1) {     // inclusive Hillis-Steele scans
    const long long a = tid >= off ? s_a[tid - off] : 0, b = tid >= off ? s_b[tid - off] : 0;
    __syncthreads();
    s_a[tid] += a;
    s_b[tid] += b;
    __syncthreads();
  }
  const long long big0 = s_a[tid] - nbig, small0 = s_b[tid] - small;
  const bool round_robin = s_a[kBalThreads - 1] == 0;
  if (tid == 0) seg_beg[kMaxBwdCtas] = round_robin ? 1 : 0;
  if (round_robin) return;                             // uniform for the block
  // big segments round-robin, and the load they put on each CTA
  long long r = big0;
  for (int64_t i = lo; i < hi; ++i) {
    const long long t = tile_off[i + 1] - tile_off[i];
    if (t >= big) atomicAdd(&load[(int)(r++ % ncta)], (int)t);
  }
  __syncthreads();
  if (tid == 0) {                                      // room left per CTA, as a prefix
    cap_off[0] = 0;
    for (int c = 0; c < ncta; ++c) {
      const long long room = fair - load[c];
      cap_off[c + 1] = cap_off[c] + (room > 0 ? room : 0);
    }
  }
  __syncthreads();
  // each segment's CTA (big: its round-robin CTA; small: the CTA whose room covers the
  // segment's first tile among the small ones)
  auto owner = [&](int64_t i, long long& rb, long long& ps) -> int {
    const long long t = tile_off[i + 1] - tile_off[i];
    if (t >= big) return (int)(rb++ % ncta);
    int a = 0, b = ncta - 1;                         // last c with cap_off[c] <= ps
    while (a < b) {
      const int m = (a + b + 1) / 2;
      if (cap_off[m] <= ps) a = m; else b = m - 1;
    }
    ps += t;
    return a;
  };
  r = big0;
  long long ps = small0;
  for (int64_t i = lo; i < hi; ++i)
    if (tile_off[i + 1] > tile_off[i]) atomicAdd(&cnt[owner(i, r, ps)], 1);
    else owner(i, r, ps);
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int c = 0; c < ncta; ++c) { seg_beg[c] = acc; acc += cnt[c]; }
    seg_beg[ncta] = acc;
  }
  __syncthreads();
  r = big0;
  ps = small0;
  for (int64_t i = lo; i < hi; ++i) {
    const bool nonempty = tile_off[i + 1] > tile_off[i];
    const int c = owner(i, r, ps);
    if (nonempty) seg_list[seg_beg[c] + atomicAdd(&fill[c], 1)] = (int)i;
  }
}

// D[b, h, t] = dO[b, t, h, :] . O[b, t, h, :] in fp32; 16 threads per row.
__global__ void bwd_dot_kernel(const __nv_bfloat16* __restrict__ dO,
                               const __nv_bfloat16* __restrict__ O, float* __restrict__ Dd,
                               int64_t rows, int hq, int64_t S) {
  const int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 16;
  const int l = threadIdx.x % 16;
  const bool live = r < rows;                          // every lane stays for the shuffles
  const uint4 z = make_uint4(0, 0, 0, 0);
  const uint4 a = live ? ldg16(dO + r * kD + l * 8) : z, c = live ? ldg16(O + r * kD + l * 8) : z;
  float fa[8], fc[8];
  Vec16<__nv_bfloat16>::unpack(a, fa);
  Vec16<__nv_bfloat16>::unpack(c, fc);
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) acc = fmaf(fa[e], fc[e], acc);
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o, 16);
  if (live && l == 0) {
    const int64_t bt = r / hq, h = r % hq;
    const int64_t b = bt / S, t = bt % S;
    Dd[(b * hq + h) * S + t] = acc;
  }
}

// ------------------------------------------------------------------ the tile kernel
constexpr int kBwdThreads = 320;      // warps 0-7 rows (softmax, epilogues), 8 MMA, 9 copies
constexpr int kIssuer = 8;
constexpr int kGather = 9;

struct __align__(8) BBars {
  uint64_t kv_full, q_full[2], q_empty[2], sdp, pds, dq, s_free, acc_empty, meta_full, meta_free;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

struct SegId {
  int b, gg, j, sub;
};
__device__ __forceinline__ SegId seg_id(int64_t s, const BGeom& g) {
  const int64_t nbs = g.nb * g.nsub;
  const int bg = (int)(s / nbs);
  const int js = (int)(s - (int64_t)bg * nbs);
  SegId d;
  d.j = js / g.nsub;
  d.sub = js - d.j * g.nsub;
  d.b = bg / g.hkv;
  d.gg = bg - d.b * g.hkv;
  return d;
}

template <int G>
__global__ void __launch_bounds__(kBwdThreads, 1)
attn_bwd_tiles_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmDO, const int4* __restrict__ tiles,
                      const int* __restrict__ tile_off, const int* __restrict__ entries,
                      const int* __restrict__ seg_list, const int* __restrict__ seg_beg,
                      const float* __restrict__ lse, const float* __restrict__ Dd,
                      __nv_bfloat16* __restrict__ dq_part, float* __restrict__ dk,
                      float* __restrict__ dv, int* err, BGeom g) {
  // this CTA's segments: the round-robin stride, or its list (bwd_balance_kernel)
  const bool rr = seg_beg[kMaxBwdCtas] != 0;
  const int64_t s_first = rr ? (int64_t)blockIdx.x : (int64_t)seg_beg[blockIdx.x];
  const int64_t s_last = rr ? g.nseg : (int64_t)seg_beg[blockIdx.x + 1];
  const int64_t s_step = rr ? (int64_t)gridDim.x : 1;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* Ks = base;                      // the segment's 128 keys   [key][d]
  unsigned char* Vs = Ks + kTile;                // and values               [key][d]
  unsigned char* Qs = Vs + kTile;                // 2 stages of query rows   [row][d]
  unsigned char* DOs = Qs + 2 * kTile;           // 2 stages of dO rows      [row][d]
  unsigned char* DSs = DOs + 2 * kTile;          // dS of the tile           [key][row]
  float* m_lse = reinterpret_cast<float*>(DSs + kTile);   // per row: lse * log2(e)
  float* m_dd = m_lse + kRowsT;                            // per row: D = dO . O
  uint8_t* m_lim = reinterpret_cast<uint8_t*>(m_dd + kRowsT);   // per row: keys it reads
  BBars* bars = reinterpret_cast<BBars*>(m_lim + kRowsT);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;

  // rows of a tile past its entries are never loaded: start from zeros, so the products
  // with their zero P and dS stay zero
  for (int i = tid; i < (int)(4 * kTile / 16); i += kBwdThreads)
    reinterpret_cast<uint4*>(Qs)[i] = make_uint4(0, 0, 0, 0);
  if (tid == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int st = 0; st < 2; ++st) {
      mbar_init(&bars->q_full[st], 1);
      mbar_init(&bars->q_empty[st], 1);
    }
    mbar_init(&bars->sdp, 1);
    mbar_init(&bars->pds, 256);
    mbar_init(&bars->dq, 1);
    mbar_init(&bars->s_free, 256);
    mbar_init(&bars->acc_empty, 256);
    mbar_init(&bars->meta_full, 128);                 // threads 0-127 publish the row data
    mbar_init(&bars->meta_free, 256);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) { tmem_alloc(&bars->tmem_base, 512); tmem_relinquish(); }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort;
  auto fail = [&]() {
    set_device_error(err, MSA_DEVERR_TIMEOUT);
    *abort_flag = 1;
  };

  if (warp == kGather) {
    // ---------------------------------------------------------------- copies
    constexpr int kTok = kRowsT / G;
    constexpr int kPerLane = (kTok + 31) / 32;
    if (lane == 0) { prefetch_tmap(&tmK); prefetch_tmap(&tmV); prefetch_tmap(&tmQ); prefetch_tmap(&tmDO); }
    int n = 0;
    bool stop = false;
    int ent_next[kPerLane];
    for (int64_t si = s_first; si < s_last && !stop; si += s_step) {
      const int64_t s = rr ? si : seg_list[si];
      const int ta = tile_off[s], tb = tile_off[s + 1];
      if (ta == tb) continue;
      const SegId id = seg_id(s, g);
      for (int tile = ta; tile < tb; ++tile, ++n) {
        if (__any_sync(0xffffffffu, *abort_flag != 0)) { stop = true; break; }
        const int st = n & 1;
        // this stage's previous tile (n - 2) and, at a segment's start, the tile before
        // (the last reader of K and V) must have finished their MMAs
        if (n >= 2 && !mbar_wait_warp(&bars->q_empty[st], (uint32_t)((n - 2) >> 1) & 1)) {
          if (lane == 0) fail();
          stop = true;
          break;
        }
        if (tile == ta && n >= 1 &&
            !mbar_wait_warp(&bars->q_empty[st ^ 1], (uint32_t)((n - 1) >> 1) & 1)) {
          if (lane == 0) fail();
          stop = true;
          break;
        }
        if (tile == ta && lane == 0) {                 // the segment's keys and values
          const int y0 = (int)((int64_t)id.b * g.S + (int64_t)id.j * g.block + (int64_t)id.sub * kSeg);
          mbar_arrive_expect_tx(&bars->kv_full, 4 * kHalf);
          for (int hf = 0; hf < 2; ++hf) {
            const int x = id.gg * kD + hf * 64;
            tma_load_2d(Ks + hf * kHalf, &tmK, &bars->kv_full, x, y0);
            tma_load_2d(Vs + hf * kHalf, &tmV, &bars->kv_full, x, y0);
          }
        }
        if (tile == ta) {                              // a segment's first tile: load it
          const int4 t0 = tiles[tile];
#pragma unroll
          for (int u = 0; u < kPerLane; ++u) {
            const int i = lane + u * 32;
            ent_next[u] = (i < kTok && i < t0.z) ? entries[t0.y + i] : -1;
          }
        }
        int ent[kPerLane];
        int n_valid = 0;
#pragma unroll
        for (int u = 0; u < kPerLane; ++u) {
          ent[u] = ent_next[u];
          n_valid += __popc(__ballot_sync(0xffffffffu, ent[u] >= 0));
        }
        if (lane == 0)
          mbar_arrive_expect_tx(&bars->q_full[st], (uint32_t)(n_valid * G * kD * 2 * 2));
        __syncwarp();
        unsigned char* qd = Qs + st * kTile;
        unsigned char* od = DOs + st * kTile;
#pragma unroll
        for (int u = 0; u < kPerLane; ++u) {
          if (ent[u] < 0) continue;
          const int i = lane + u * 32;
          const int y = (int)(((int64_t)id.b * g.S + (ent[u] >> 6)) * g.hq + id.gg * G);
          tma_load_2d(qd + i * G * 128, &tmQ, &bars->q_full[st], 0, y);
          tma_load_2d(qd + kHalf + i * G * 128, &tmQ, &bars->q_full[st], 64, y);
          tma_load_2d(od + i * G * 128, &tmDO, &bars->q_full[st], 0, y);
          tma_load_2d(od + kHalf + i * G * 128, &tmDO, &bars->q_full[st], 64, y);
        }
        // the next tile of the segment: its entries kept for the next iteration's copies
        // (an L2 prefetch of its rows was measured 31% slower: the tile kernel is bound by
        // the rate of small tensor-map operations)
        if (tile + 1 < tb) {
          const int4 tn = tiles[tile + 1];
#pragma unroll
          for (int u = 0; u < kPerLane; ++u) {
            const int i = lane + u * 32;
            ent_next[u] = (i < kTok && i < tn.z) ? entries[tn.y + i] : -1;
          }
        }
      }
    }
    // nothing may still be landing when the CTA exits
    for (int m = n >= 2 ? n - 2 : 0; m < n; ++m)
      if (!mbar_wait_warp(&bars->q_empty[m & 1], (uint32_t)(m >> 1) & 1)) break;
  } else if (warp == kIssuer) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      const uint32_t idKK = idesc_bf16(128, 128, 0, 0);   // S^T, dP^T: both operands K-major
      const uint32_t idTM = idesc_bf16(128, 128, 0, 1);   // dV, dK: A = P^T / dS^T in TMEM
      const uint32_t idMM = idesc_bf16(128, 128, 1, 1);   // dQ: A = dS MN-major
      const uint64_t kk = sdesc_sw128(smem_u32(Ks), 16, 1024), kv = sdesc_sw128(smem_u32(Vs), 16, 1024);
      const uint64_t kq0 = sdesc_sw128(smem_u32(Qs), 16, 1024), kdo0 = sdesc_sw128(smem_u32(DOs), 16, 1024);
      const uint64_t mq0 = sdesc_sw128(smem_u32(Qs), kHalf, 1024), mdo0 = sdesc_sw128(smem_u32(DOs), kHalf, 1024);
      const uint64_t mk = sdesc_sw128(smem_u32(Ks), kHalf, 1024), mds = sdesc_sw128(smem_u32(DSs), kHalf, 1024);
      constexpr uint64_t kStage = kTile >> 4;            // descriptor units between stages
      auto koff = [](int ks) -> uint64_t {             // K-major: 16 elements of the d axis
        return (uint64_t)((ks >> 2) * (kHalf >> 4) + (ks & 3) * 2);
      };
      auto moff = [](int ks) -> uint64_t { return (uint64_t)ks * (2048 >> 4); };  // 16 K-rows
      int n = 0, sc = 0;
      bool ok = true;
      for (int64_t si = s_first; si < s_last && ok; si += s_step) {
        const int64_t s = rr ? si : seg_list[si];
        const int ta = tile_off[s], tb = tile_off[s + 1];
        if (ta == tb) continue;
        if (!mbar_wait(&bars->kv_full, (uint32_t)sc & 1)) { ok = false; break; }
        for (int tile = ta; tile < tb; ++tile, ++n) {
          if (*abort_flag) { ok = false; break; }
          const int st = n & 1;
          if (!mbar_wait(&bars->q_full[st], (uint32_t)(n >> 1) & 1)) { ok = false; break; }
          if (n > 0 && !mbar_wait(&bars->s_free, (uint32_t)(n - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint64_t kq = kq0 + st * kStage, kdo = kdo0 + st * kStage;
          const uint64_t mq = mq0 + st * kStage, mdo = mdo0 + st * kStage;
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) umma_ss(tmem + 0, kk + koff(ks), kq + koff(ks), idKK, ks > 0);
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) umma_ss(tmem + 128, kv + koff(ks), kdo + koff(ks), idKK, ks > 0);
          umma_commit(&bars->sdp);
          if (!mbar_wait(&bars->pds, (uint32_t)n & 1)) { ok = false; break; }
          if (tile == ta && sc > 0 && !mbar_wait(&bars->acc_empty, (uint32_t)(sc - 1) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t first = tile == ta ? 1u : 0u;
          // P^T / dS^T as packed bf16: rows 16 ks.. at column 8 ks, plus 32 for rows 64..127
          // (each half of the rows is packed into the columns its threads read)
#pragma unroll
          for (int ks = 0; ks < kRowsT / 16; ++ks)
            umma_ts(tmem + 256, tmem + 0 + ks * 8 + (ks >= 4 ? 32 : 0), mdo + moff(ks), idTM,
                    (first && ks == 0) ? 0u : 1u);
#pragma unroll
          for (int ks = 0; ks < kRowsT / 16; ++ks)
            umma_ts(tmem + 384, tmem + 128 + ks * 8 + (ks >= 4 ? 32 : 0), mq + moff(ks), idTM,
                    (first && ks == 0) ? 0u : 1u);
          // dQ over S^T's columns: the MMAs of this thread run in issue order, so the dV
          // products above have read P^T from them before these write
#pragma unroll
          for (int ks = 0; ks < kSeg / 16; ++ks) umma_ss(tmem + 0, mds + moff(ks), mk + moff(ks), idMM, ks > 0);
          umma_commit(&bars->dq);
          umma_commit(&bars->q_empty[st]);
        }
        ++sc;
      }
      if (!ok) fail();
    }
  } else {
    // ---------------------------------------------------------------- rows (warps 0-7)
    // Thread tid covers tile row r = tid % 128 for the per-row data (threads 0-127 publish
    // it) and the dQ epilogue (d half hf = tid / 128), and key r (TMEM lane r of S^T, dP^T,
    // dV, dK) for the softmax over rows [64 hf, 64 hf + 64) and the dV / dK epilogue of
    // d half hf.  Two threads per lane keep eight warps on the elementwise work.
    const int r = tid & (kRowsT - 1), hf = tid >> 7;
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const int i_tok = r / G, h = r % G;
    const float c2 = g.scale_log2;
    const uint32_t sDS = smem_u32(DSs);
    int n = 0;
    bool ok = true;
    for (int64_t si = s_first; si < s_last && ok; si += s_step) {
      const int64_t s = rr ? si : seg_list[si];
      const int ta = tile_off[s], tb = tile_off[s + 1];
      if (ta == tb) continue;
      const SegId id = seg_id(s, g);
      const int64_t kbase = (int64_t)id.j * g.block + (int64_t)id.sub * kSeg;
      const int64_t seg_end = min(min((int64_t)id.j * g.block + g.block, kbase + kSeg), g.S);
      // row r of a tile: its entry, and its lse and D (loaded one tile ahead)
      auto row_of = [&](int e, float& lse_o, float& dd_o) {
        if (e < 0) { lse_o = 0.f; dd_o = 0.f; return; }
        const int64_t hr = ((int64_t)id.b * g.hq + id.gg * G + h) * g.S + (e >> 6);
        lse_o = lse[hr] * kLog2e;
        dd_o = Dd[hr];
      };
      int4 tl_next = tiles[ta];
      int ent_next = i_tok < tl_next.z ? entries[tl_next.y + i_tok] : -1;
      float lse_next, dd_next;
      row_of(hf == 0 ? ent_next : -1, lse_next, dd_next);
      for (int tile = ta; tile < tb; ++tile, ++n) {
        if (__any_sync(0xffffffffu, *abort_flag != 0)) { ok = false; break; }
        const int ent = ent_next;
        const float lse_r = lse_next, dd_r = dd_next;
        if (tile + 1 < tb) tl_next = tiles[tile + 1];
        const bool valid = ent >= 0;
        const int64_t t = valid ? (ent >> 6) : 0;
        const int pslot = valid ? (ent & 63) : 0;
        int64_t end = seg_end;
        if (valid && t / g.block == id.j) end = min(end, t + 1);     // causal, own block
        const int lim = valid ? (int)max((int64_t)0, end - kbase) : 0;
        // row r's data for every key thread, once the previous tile's readers are done
        // with it (bounded mbarrier waits: a warp that gives up cannot strand the others)
        if (n > 0 && !mbar_wait_warp(&bars->meta_free, (uint32_t)(n - 1) & 1)) { ok = false; break; }
        if (hf == 0) {
          m_lse[r] = lse_r;
          m_dd[r] = dd_r;
          m_lim[r] = (uint8_t)lim;
          mbar_arrive(&bars->meta_full);
        }
        if (!mbar_wait_warp(&bars->meta_full, (uint32_t)n & 1)) { ok = false; break; }
        if (!mbar_wait_warp(&bars->sdp, (uint32_t)n & 1)) { ok = false; break; }
        tc_fence_after();
        if (tile + 1 < tb) {
          ent_next = i_tok < tl_next.z ? entries[tl_next.y + i_tok] : -1;
          row_of(hf == 0 ? ent_next : -1, lse_next, dd_next);
        }
        // key r: P^T and dS^T over rows [64 hf, 64 hf + 64), back into TMEM as bf16 (A
        // operands of dV and dK), and dS into shared memory ([key][row], A of dQ)
#pragma unroll 1
        for (int c = 2 * hf; c < 2 * hf + 2; ++c) {
          uint32_t sv[32], pv[32];
          tmem_ld32(lane_base + c * 32, sv);
          tmem_ld32(lane_base + 128 + c * 32, pv);
          tmem_ld_wait();
          uint32_t pp[16], pd[16];
#pragma unroll
          for (int k = 0; k < 32; k += 4) {
            const int rr = c * 32 + k;
            const float4 l4 = *reinterpret_cast<const float4*>(m_lse + rr);
            const float4 d4 = *reinterpret_cast<const float4*>(m_dd + rr);
            const uint32_t lim4 = *reinterpret_cast<const uint32_t*>(m_lim + rr);
            const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dvv[4] = {d4.x, d4.y, d4.z, d4.w};
            float p[4], ds[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int lim_e = (int)((lim4 >> (8 * e)) & 0xffu);
              p[e] = r < lim_e ? fastmath::fast_exp2(__uint_as_float(sv[k + e]) * c2 - lv[e]) : 0.f;
              ds[e] = p[e] * (__uint_as_float(pv[k + e]) - dvv[e]) * g.scale;
            }
            pp[k / 2] = pack_bf16x2(p[0], p[1]);
            pp[k / 2 + 1] = pack_bf16x2(p[2], p[3]);
            pd[k / 2] = pack_bf16x2(ds[0], ds[1]);
            pd[k / 2 + 1] = pack_bf16x2(ds[2], ds[3]);
          }
          // packed bf16 pairs over S^T / dP^T columns this thread has already read: rows
          // 32c.. of half 0 at column 16c, of half 1 at 64 + 16(c - 2)
          const uint32_t colp = (uint32_t)(c * 16 + (c >= 2 ? 32 : 0));
          tmem_st16(lane_base + colp, pp);
          tmem_st16(lane_base + 128 + colp, pd);
          const uint32_t half = (uint32_t)(c >> 1) * kHalf + (uint32_t)r * 128;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const uint32_t chunk = (uint32_t)((c & 1) * 4 + c4);
            const uint32_t off = half + ((chunk ^ (uint32_t)(r & 7)) << 4);
            st_shared_v4(sDS + off, pd[c4 * 4], pd[c4 * 4 + 1], pd[c4 * 4 + 2], pd[c4 * 4 + 3]);
          }
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars->pds);
        mbar_arrive(&bars->meta_free);                 // this thread is done with the row data
        if (!mbar_wait_warp(&bars->dq, (uint32_t)n & 1)) { ok = false; break; }
        tc_fence_after();
        // row r's dQ partial, d half hf (lane r of the dQ accumulator), bf16, 32-byte stores
        const int64_t prow = ((int64_t)(id.b * g.hkv + id.gg)) * g.slab + (t - g.t_base);
        __nv_bfloat16* dst = dq_part + ((prow * g.kslots + pslot) * G + h) * kD;
#pragma unroll 1
        for (int kc = 2 * hf; kc < 2 * hf + 2; ++kc) {
          uint32_t qv[32];
          tmem_ld32(lane_base + kc * 32, qv);
          tmem_ld_wait();
          uint32_t ob[16];
#pragma unroll
          for (int k = 0; k < 32; k += 2)
            ob[k / 2] = pack_bf16x2(__uint_as_float(qv[k]), __uint_as_float(qv[k + 1]));
          if (valid) {
            st_global_v8(dst + kc * 32, ob);
            st_global_v8(dst + kc * 32 + 16, ob + 8);
          }
        }
        tc_fence_before();
        mbar_arrive(&bars->s_free);
        if (tile == tb - 1) {
          // the segment's dV and dK are complete (the commit covered every earlier MMA):
          // lane r = key kbase + r, d half hf, added to the fp32 gradients
          const int64_t key = kbase + r;
          const bool kvalid = key < seg_end;
#pragma unroll 1
          for (int which = 0; which < 2; ++which) {
            float* outp = (which == 0 ? dv : dk) + (((int64_t)id.b * g.S + key) * g.hkv + id.gg) * kD;
#pragma unroll 1
            for (int kc = 2 * hf; kc < 2 * hf + 2; ++kc) {
              uint32_t av[32];
              tmem_ld32(lane_base + 256 + which * 128 + kc * 32, av);
              tmem_ld_wait();
              if (kvalid) {
#pragma unroll
                for (int k = 0; k < 32; k += 4) {
                  float4* o4 = reinterpret_cast<float4*>(outp + kc * 32 + k);
                  float4 x = *o4;
                  x.x += __uint_as_float(av[k]);
                  x.y += __uint_as_float(av[k + 1]);
                  x.z += __uint_as_float(av[k + 2]);
                  x.w += __uint_as_float(av[k + 3]);
                  *o4 = x;
                }
              }
            }
          }
          tc_fence_before();
          mbar_arrive(&bars->acc_empty);
        }
      }
    }
    if (!ok) fail();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// dQ[b, t, g*G + h, :] = sum over the row's (slot, segment) partials, in slot order.
template <int G>
__global__ void __launch_bounds__(128)
bwd_merge_dq_kernel(const int32_t* __restrict__ idx, const __nv_bfloat16* __restrict__ part,
                    float* __restrict__ dq, BGeom g, int64_t n_rows) {
  constexpr int TPR = G * 8;                           // 16 elements per thread
  constexpr int RPC = 128 / TPR;
  const int64_t row = (int64_t)blockIdx.x * RPC + threadIdx.x / TPR;
  if (row >= n_rows) return;
  const int lt = threadIdx.x % TPR;
  const int64_t bg = row / g.slab;
  const int t = (int)(g.t_base + row % g.slab);
  if (t >= g.t_end) return;
  const int64_t gg = bg % g.hkv, b = bg / g.hkv;
  const int own = t / (int)g.block;
  const int32_t* irow = idx + (bg * g.S + t) * g.topk;
  const __nv_bfloat16* prow = part + row * g.kslots * G * kD + lt * 16;
  float acc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] = 0.f;
  for (int sl = 0; sl < g.topk; ++sl) {
    const int j = irow[sl];
    if (j < 0 || j >= g.nb || j > own) continue;
    for (int sub = 0; sub < g.nsub; ++sub) {
      if (!seg_has_keys(j, own, t, sub, g)) continue;
      const uint4* src = reinterpret_cast<const uint4*>(prow + (int64_t)(sl * g.nsub + sub) * G * kD);
      float f[8];
      Vec16<__nv_bfloat16>::unpack(src[0], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += f[e];
      Vec16<__nv_bfloat16>::unpack(src[1], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[8 + e] += f[e];
    }
  }
  float* dst = dq + ((b * g.S + t) * g.hq + gg * G) * kD + lt * 16;
#pragma unroll
  for (int e = 0; e < 16; e += 4)
    *reinterpret_cast<float4*>(dst + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
}

// ------------------------------------------------------------------ host side
struct BLayout {
  size_t counts, totals, seg_off, tile_off, n_tiles, entries, tiles, part, dd, seg_list,
      seg_beg, total;
};

size_t up256b(size_t x) { return (x + 255) / 256 * 256; }

BGeom make_bgeom(const Shape& s) {
  BGeom g{};
  g.S = s.seq; g.nb = s.nb; g.block = s.block;
  g.hq = (int)s.hq; g.hkv = (int)s.hkv; g.G = (int)(s.hq / s.hkv); g.topk = (int)s.topk;
  g.nsub = (int)((s.block + kSeg - 1) / kSeg);
  g.kslots = g.topk * g.nsub;
  g.tpt = kRowsT / g.G;
  g.nseg = s.batch * s.hkv * s.nb * g.nsub;
  g.scale = s.scale;
  g.scale_log2 = s.scale * kLog2e;
  g.t_base = 0; g.t_end = s.seq; g.slab = s.seq;
  g.n_ranges = (int)((s.seq + kTokRange - 1) / kTokRange);
  return g;
}

BLayout blayout(const Shape& s, int64_t slab) {
  BGeom g = make_bgeom(s);
  const int64_t ranges = (slab + kTokRange - 1) / kTokRange;
  const int64_t n_entries = s.batch * s.hkv * slab * s.topk * g.nsub;
  const int64_t n_tiles_max = n_entries / g.tpt + g.nseg + 1;
  const int64_t rows = s.batch * s.hkv * slab;
  BLayout L{};
  size_t o = 0;
  L.counts = o;   o += up256b((size_t)s.batch * s.hkv * ranges * s.nb * g.nsub * 4);
  L.totals = o;   o += up256b((size_t)g.nseg * 4);
  L.seg_off = o;  o += up256b((size_t)(g.nseg + 1) * 4);
  L.tile_off = o; o += up256b((size_t)(g.nseg + 1) * 4);
  L.n_tiles = o;  o += 256;
  L.entries = o;  o += up256b((size_t)n_entries * 4);
  L.tiles = o;    o += up256b((size_t)n_tiles_max * 16);
  L.part = o;     o += up256b((size_t)rows * g.kslots * g.G * kD * 2);
  L.dd = o;       o += up256b((size_t)s.batch * s.hq * s.seq * 4);
  L.seg_list = o; o += up256b((size_t)g.nseg * 4);
  L.seg_beg = o;  o += up256b((size_t)(kMaxBwdCtas + 1) * 4);
  L.total = o;
  return L;
}

constexpr size_t kBwdSlabBudget = (size_t)32 << 30;
int64_t bwd_slab_for(const Shape& s, size_t bytes) {
  if (blayout(s, s.seq).total <= bytes) return s.seq;
  int64_t lo = 1, hi = s.seq / kTokRange;
  if (hi < 1) return s.seq;
  while (lo < hi) {
    const int64_t mid = (lo + hi + 1) / 2;
    if (blayout(s, mid * kTokRange).total <= bytes) lo = mid; else hi = mid - 1;
  }
  const int64_t units = (s.seq + kTokRange - 1) / kTokRange;
  const int64_t n_slabs = (units + lo - 1) / lo;
  return (units + n_slabs - 1) / n_slabs * kTokRange;
}

template <int G>
cudaError_t run_bwd(const Shape& s, const BGeom& g, const CUtensorMap& mk, const CUtensorMap& mv,
                    const CUtensorMap& mq, const CUtensorMap& mdo, const int32_t* idx,
                    const float* lse, float* dq, float* dk, float* dv, char* ws, const BLayout& L,
                    int* err, cudaStream_t st) {
  const size_t smem = 1024 + 7 * (size_t)kTile + kRowsT * (4 + 4 + 1) + sizeof(BBars);
  static_assert(1024 + 7 * (size_t)kTile + kRowsT * (4 + 4 + 1) + sizeof(BBars) <= 232448,
                "backward tile kernel exceeds 227 KB of shared memory");
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_tiles_kernel<G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int grid = sm_count();
  if (g.nseg < grid) grid = (int)g.nseg;
  if (grid > kMaxBwdCtas - 1) grid = kMaxBwdCtas - 1;      // seg_beg[kMaxBwdCtas] is the mode
  bwd_balance_kernel<<<1, kBalThreads, 0, st>>>((const int*)(ws + L.tile_off), g.nseg, grid,
                                                (int*)(ws + L.seg_list), (int*)(ws + L.seg_beg));
  attn_bwd_tiles_kernel<G><<<grid, kBwdThreads, smem, st>>>(
      mk, mv, mq, mdo, (const int4*)(ws + L.tiles), (const int*)(ws + L.tile_off),
      (const int*)(ws + L.entries), (const int*)(ws + L.seg_list),
      (const int*)(ws + L.seg_beg), lse, (const float*)(ws + L.dd),
      (__nv_bfloat16*)(ws + L.part), dk, dv, err, g);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t rows = s.batch * s.hkv * g.slab;
  const int rpc = 128 / (G * 8);
  bwd_merge_dq_kernel<G><<<(unsigned)((rows + rpc - 1) / rpc), 128, 0, st>>>(
      idx, (const __nv_bfloat16*)(ws + L.part), dq, g, rows);
  return cudaGetLastError();
}

}  // namespace

bool tc_attn_bwd_supported(const Shape& s) {
  if (s.dtype != MSA_BF16 || s.d != kD) return false;
  if (s.block % kSeg != 0) return false;
  const int64_t G = s.hq / s.hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return false;
  const int64_t nsub = s.block / kSeg;
  if (s.topk * nsub > 64) return false;                        // pslot fits 6 bits
  if (s.seq >= ((int64_t)1 << 25)) return false;               // token fits 25 bits
  if (s.batch * s.seq * s.hq >= ((int64_t)1 << 31)) return false;
  if (s.batch * s.hkv * s.seq * s.topk * nsub >= ((int64_t)1 << 31)) return false;
  if (s.nb * nsub > 40 * 1024) return false;                   // per-segment counters in smem
  return true;
}

size_t tc_attn_bwd_ws_bytes(const Shape& s) { return blayout(s, bwd_slab_for(s, kBwdSlabBudget)).total; }
size_t tc_attn_bwd_ws_min_bytes(const Shape& s) {
  return blayout(s, s.seq < kTokRange ? s.seq : kTokRange).total;
}

cudaError_t launch_attn_bwd_tc(const Shape& s, const void* q, const void* k, const void* v,
                               const void* o, const float* lse, const void* dout,
                               const int32_t* idx, float* dq, float* dk, float* dv, void* ws_body,
                               size_t ws_body_bytes, int* err, cudaStream_t st) {
  BGeom g = make_bgeom(s);
  const int64_t slab = bwd_slab_for(s, ws_body_bytes);
  const BLayout L = blayout(s, slab);
  if (L.total > ws_body_bytes) return cudaErrorInvalidValue;
  g.slab = slab;
  char* ws = reinterpret_cast<char*>(ws_body);
  CUtensorMap mk, mv, mq, mdo;
  if (!make_bf16_2d_map(&mk, k, s.batch * s.seq, s.hkv * kD, kSeg) ||
      !make_bf16_2d_map(&mv, v, s.batch * s.seq, s.hkv * kD, kSeg) ||
      !make_bf16_2d_map(&mq, q, s.batch * s.seq * s.hq, kD, g.G) ||
      !make_bf16_2d_map(&mdo, dout, s.batch * s.seq * s.hq, kD, g.G))
    return cudaErrorInvalidValue;
  cudaError_t e;
  const size_t gsz = (size_t)s.batch * s.seq * s.hkv * kD * sizeof(float);
  if ((e = cudaMemsetAsync(dk, 0, gsz, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(dv, 0, gsz, st)) != cudaSuccess) return e;
  const int64_t rows_all = s.batch * s.seq * s.hq;
  bwd_dot_kernel<<<(unsigned)((rows_all * 16 + 255) / 256), 256, 0, st>>>(
      (const __nv_bfloat16*)dout, (const __nv_bfloat16*)o, (float*)(ws + L.dd), rows_all,
      (int)s.hq, s.seq);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t hsmem = (size_t)g.nb * g.nsub * sizeof(int);
  if ((e = cudaFuncSetAttribute(bwd_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)hsmem)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(bwd_fill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)hsmem)) != cudaSuccess)
    return e;
  for (int64_t t0 = 0; t0 < s.seq; t0 += slab) {
    g.t_base = t0;
    g.t_end = t0 + slab < s.seq ? t0 + slab : s.seq;
    g.n_ranges = (int)((g.t_end - t0 + kTokRange - 1) / kTokRange);
    const dim3 rgrid((unsigned)g.n_ranges, (unsigned)(s.batch * s.hkv));
    bwd_count_kernel<<<rgrid, 512, hsmem, st>>>(idx, (int*)(ws + L.counts), err, g);
    bwd_colscan_kernel<<<(unsigned)((g.nseg + 255) / 256), 256, 0, st>>>(
        (int*)(ws + L.counts), (int*)(ws + L.totals), g);
    bwd_scan_kernel<<<1, 1024, 0, st>>>((const int*)(ws + L.totals), (int*)(ws + L.seg_off),
                                        (int*)(ws + L.tile_off), (int*)(ws + L.n_tiles), g.nseg,
                                        g.tpt);
    bwd_fill_kernel<<<rgrid, 32, hsmem, st>>>(idx, (const int*)(ws + L.counts),
                                              (const int*)(ws + L.seg_off), (int*)(ws + L.entries),
                                              g);
    const int64_t n_sel = s.batch * s.hkv * (g.t_end - t0) * s.topk;
    const int64_t n_tiles_max = n_sel * g.nsub / g.tpt + g.nseg + 1;
    bwd_tile_table_kernel<<<(unsigned)((n_tiles_max + 255) / 256), 256, 0, st>>>(
        (const int*)(ws + L.totals), (const int*)(ws + L.seg_off), (const int*)(ws + L.tile_off),
        (const int*)(ws + L.n_tiles), (int4*)(ws + L.tiles), g.nseg, g.tpt,
        (int64_t)g.nb * g.nsub);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    switch (g.G) {
      case 1: e = run_bwd<1>(s, g, mk, mv, mq, mdo, idx, lse, dq, dk, dv, ws, L, err, st); break;
      case 2: e = run_bwd<2>(s, g, mk, mv, mq, mdo, idx, lse, dq, dk, dv, ws, L, err, st); break;
      case 4: e = run_bwd<4>(s, g, mk, mv, mq, mdo, idx, lse, dq, dk, dv, ws, L, err, st); break;
      default: e = run_bwd<8>(s, g, mk, mv, mq, mdo, idx, lse, dq, dk, dv, ws, L, err, st); break;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace msa
