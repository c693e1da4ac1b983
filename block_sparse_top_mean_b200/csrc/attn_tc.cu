// Step 4 on the tensor cores (bf16, d = 128): key-centric block-sparse attention.
//
// Every (token, group) selects different blocks, so query-centric tiles would share no
// keys.  Instead the selection is inverted: for each (sequence, group, block) the list
// of (token, slot) entries that selected it is built, and one tile = the G query heads
// of 128/G such tokens (128 rows) against that block's keys.  K/V of a block are loaded
// once per run of tiles into shared memory with TMA; the tile's query rows are gathered
// with tensor-map boxes (G heads of one token each) into the 128-byte-swizzled K-major
// layout the MMA reads.
//
// Per tile, per 128-key chunk c (a block of 256 keys is 2 chunks; longer blocks are
// split into 256-key segments, each its own partial slot):
//   S_c = Q K_c^T      tcgen05.mma, M=128 N=128 K=128, fp32 accumulator in TMEM
//   softmax            one thread per row reads S_c from TMEM, masks (ragged block,
//                      causal inside the own block), base-2 exponentials in fp32,
//                      writes P_c as bf16 back into TMEM over S_c
//   O_c = P_c V_c      tcgen05.mma with A from TMEM, B = V (MN-major) from shared memory
// O accumulates over the chunks in TMEM; the epilogue writes a normalised bf16 partial O
// plus its log-sum-exp for (token, slot); a second kernel merges a row's partials into O.
// TMEM columns: S/P of tile parity 0 [0,128), 1 [128,256); O of parity 0 [256,384),
// 1 [384,512).
#include <cudaTypedefs.h>
#include <math_constants.h>

#include "common.cuh"
#include "fastmath.cuh"
#include "sm100.cuh"

namespace msa {
namespace {

using namespace sm100;
using namespace fastmath;

constexpr int kD = 128;
constexpr int kRowsT = 128;          // rows per tile
constexpr int kChunkKeys = 128;      // keys per MMA chunk
constexpr int kSegKeys = 256;        // keys per segment
constexpr uint32_t kTileBytes = 16384;   // 128 rows x 128 B
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct Geom {
  int64_t S, nb, block, nseg;
  int64_t t_base, t_end, slab;   // this call's token slab [t_base, t_end); partial rows per (b, g)
  int hq, hkv, G, topk, nsub, kslots, tpt, nch;
  float scale_log2;
};

// ------------------------------------------------------------------ index inversion
// Counting and filling run per CTA over a range of kInvTokens tokens of one (sequence,
// group): entries are first counted in a shared-memory histogram over that group's
// segments, so the global atomics are one per non-empty segment per CTA instead of one
// per entry.  The fill reserves each segment's range with one atomic and places its
// entries with shared-memory atomics.  The order of entries inside a segment is not
// defined; no row's arithmetic depends on it.
constexpr int kInvTokens = 2048;
constexpr int kInvThreads = 512;

__device__ __forceinline__ bool sub_has_keys32(int j, int own, int t, int sub, const Geom& g) {
  const int64_t lo = (int64_t)j * g.block + (int64_t)sub * kSegKeys;
  if ((int64_t)sub * kSegKeys >= g.block || lo >= g.S) return false;
  return j < own || lo <= t;
}

// FILL = false: add the CTA's counts to counts[]; FILL = true: write entries[].
template <bool FILL>
__global__ void __launch_bounds__(kInvThreads)
invert_hist_kernel(const int32_t* __restrict__ idx, int* __restrict__ counts,
                   int* __restrict__ cursor, int* __restrict__ entries, int* err, Geom g) {
  extern __shared__ int hist[];                       // nb * nsub counters
  const int nbs = (int)g.nb * g.nsub;
  const int t0 = (int)g.t_base + blockIdx.x * kInvTokens;
  const int bg = blockIdx.y;                          // sequence * hkv + group
  const int t1 = (int)min((int64_t)t0 + kInvTokens, g.t_end);
  const int own_max = (t1 - 1) / (int)g.block;        // segments beyond it stay empty
  const int used = min(nbs, (own_max + 1) * g.nsub);
  for (int i = threadIdx.x; i < used; i += kInvThreads) hist[i] = 0;
  __syncthreads();
  const int32_t* irow = idx + ((int64_t)bg * g.S + t0) * g.topk;
  const int n = (t1 - t0) * g.topk;
  for (int e = threadIdx.x; e < n; e += kInvThreads) {
    const int j = irow[e];
    if (j == -1) continue;
    const int t = t0 + e / g.topk;
    const int own = t / (int)g.block;
    if (j < -1 || j >= g.nb || j > own) {
      if (!FILL) set_device_error(err, MSA_DEVERR_IDX_RANGE);
      continue;
    }
    for (int sub = 0; sub < g.nsub; ++sub)
      if (sub_has_keys32(j, own, t, sub, g)) atomicAdd(&hist[j * g.nsub + sub], 1);
  }
  __syncthreads();
  int* gcount = (FILL ? cursor : counts) + (int64_t)bg * nbs;
  for (int i = threadIdx.x; i < used; i += kInvThreads) {
    const int c = hist[i];
    if (c == 0) continue;
    const int base = atomicAdd(&gcount[i], c);        // FILL: reserve [base, base + c)
    if (FILL) hist[i] = base;
  }
  if (!FILL) return;
  __syncthreads();
  for (int e = threadIdx.x; e < n; e += kInvThreads) {
    const int j = irow[e];
    if (j < 0 || j >= g.nb) continue;
    const int t = t0 + e / g.topk;
    const int own = t / (int)g.block;
    if (j > own) continue;
    const int slot = e % g.topk;
    for (int sub = 0; sub < g.nsub; ++sub)
      if (sub_has_keys32(j, own, t, sub, g)) {
        const int pos = atomicAdd(&hist[j * g.nsub + sub], 1);
        entries[pos] = (t << 6) | (slot * g.nsub + sub);
      }
  }
}

// Single-CTA exclusive scans: seg_off (entries), tile_off (tiles of tpt entries).
__global__ void __launch_bounds__(1024)
invert_scan_kernel(const int* __restrict__ counts, int* __restrict__ seg_off,
                   int* __restrict__ cursor, int* __restrict__ tile_off, int* __restrict__ n_tiles,
                   int64_t nseg, int tpt) {
  __shared__ long long s_e[1024], s_t[1024];
  const int tid = threadIdx.x;
  const int64_t per = (nseg + 1023) / 1024;
  const int64_t lo = tid * per, hi = lo + per < nseg ? lo + per : nseg;
  long long se = 0, st = 0;
  for (int64_t i = lo; i < hi; ++i) { se += counts[i]; st += (counts[i] + tpt - 1) / tpt; }
  s_e[tid] = se; s_t[tid] = st;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {     // Hillis-Steele inclusive scan
    long long a = tid >= off ? s_e[tid - off] : 0, b = tid >= off ? s_t[tid - off] : 0;
    __syncthreads();
    s_e[tid] += a; s_t[tid] += b;
    __syncthreads();
  }
  long long ce = s_e[tid] - se, ct = s_t[tid] - st;
  for (int64_t i = lo; i < hi; ++i) {
    seg_off[i] = (int)ce; cursor[i] = (int)ce; tile_off[i] = (int)ct;
    ce += counts[i]; ct += (counts[i] + tpt - 1) / tpt;
  }
  if (tid == 1023) { seg_off[nseg] = (int)s_e[1023]; tile_off[nseg] = (int)s_t[1023];
                     *n_tiles = (int)s_t[1023]; }
}

__global__ void tile_table_kernel(const int* __restrict__ counts, const int* __restrict__ seg_off,
                                  const int* __restrict__ tile_off,
                                  const int* __restrict__ n_tiles, int4* __restrict__ tiles,
                                  int64_t nseg, int tpt, int64_t nseg_per_bg) {
  const int64_t tile = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (tile >= *n_tiles) return;
  int64_t lo = 0, hi = nseg;                     // largest s with tile_off[s] <= tile
  while (hi - lo > 1) {
    const int64_t mid = (lo + hi) / 2;
    if (tile_off[mid] <= tile) lo = mid; else hi = mid;
  }
  while (lo + 1 < nseg && tile_off[lo + 1] <= tile) ++lo;   // skip empty segments
  const int k = (int)(tile - tile_off[lo]);
  const int cnt = min(tpt, counts[lo] - k * tpt);
  // x = segment, y = first entry, z = entries, w = sequence * hkv + group
  tiles[tile] = make_int4((int)lo, seg_off[lo] + k * tpt, cnt, (int)(lo / nseg_per_bg));
}

// ------------------------------------------------------------------ the tile kernel
// Two tiles are in flight: tile n (the n-th of this CTA) uses TMEM set X = n & 1
// (S_X at columns 128X, O_X at 256 + 128X), Q stage n % stages and softmax warpgroup X.
// The issuer runs the tiles of one block as two interleaved streams (even and odd tiles),
// so the tensor core works on one tile while the other tile's warpgroup runs its softmax
// or epilogue.  MMAs of one thread run in issue order, so a QK may reuse the TMEM of a P
// that an earlier PV reads; only thread accesses of TMEM (softmax, epilogue) and TMA
// writes of K/V wait for MMA completion.  One O accumulator per tile: chunk 1 reuses
// chunk 0's row max as its exponent reference unless the max grew by more than 2^8, in
// which case that warp rescales O in TMEM after chunk 0's PV completed.
constexpr int kMaxQStages = 4;
struct __align__(8) Bars {
  uint64_t q_full[kMaxQStages], q_empty[kMaxQStages];
  uint64_t s_full[2], p_full[2], pv_done[2], o_empty[2], kv_full;
  uint32_t tmem_base;
  int abort;
};

// Q stages: a tile holds its stage until its last chunk's QK, so 256-key blocks (two
// chunks, 128 KB of K/V) get 3 stages and 128-key blocks 4 (both fit 227 KB).
__host__ __device__ constexpr int q_stages(int nch) { return nch == 1 ? 4 : 3; }

constexpr int kThreads3 = 320;       // WG0 warps 0-3, WG1 warps 4-7, issuer 8, gather 9
constexpr int kIssuerWarp = 8;
constexpr int kGatherWarp = 9;
constexpr float kRescaleLog2 = 8.f;  // chunk-1 max may exceed the reference by 2^8


// Decodes a tile record into (sequence, group, block, 256-key segment) with 32-bit math.
struct TileId {
  int b, gg, j, sub;
};
__device__ __forceinline__ TileId decode_tile(const int4& tl, const Geom& g) {
  TileId d;
  const int nbs = (int)g.nb * g.nsub;
  const int js = tl.x - tl.w * nbs;
  d.j = js / g.nsub;
  d.sub = js - d.j * g.nsub;
  d.b = tl.w / g.hkv;
  d.gg = tl.w - d.b * g.hkv;
  return d;
}

#ifndef MSA_POLY_PAIRS
#define MSA_POLY_PAIRS 0x44                       // pairs (of 8) whose exponentials use the FMA pipe
#endif

// Phase parity of the per-chunk barriers for chunk c of this CTA's tile n.
__device__ __forceinline__ uint32_t chunk_phase(int n, int c, int nch) {
  return (uint32_t)(((n >> 1) * nch + c) & 1);
}

template <int G>
__global__ void __launch_bounds__(kThreads3, 1)
attn_tiles_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmQ, const int4* __restrict__ tiles,
                  const int* __restrict__ n_tiles_p, const int* __restrict__ entries,
                  __nv_bfloat16* __restrict__ po, float* __restrict__ plse, int* err, Geom g) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nch = g.nch;
  const int nqs = q_stages(nch);
  unsigned char* Qs = base;                                   // nqs stages x 32 KB
  unsigned char* Ks = base + nqs * 2 * kTileBytes;            // nch x 2 halves x 16 KB
  unsigned char* Vs = Ks + nch * 2 * kTileBytes;
  Bars* bars = reinterpret_cast<Bars*>(Vs + nch * 2 * kTileBytes);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int n_tiles = *n_tiles_p;
  const int per = (n_tiles + gridDim.x - 1) / gridDim.x;
  const int tile_lo = blockIdx.x * per;
  const int tile_hi = min(n_tiles, tile_lo + per);
  const int my_tiles = max(0, tile_hi - tile_lo);

  if (tid == 0) {
    for (int s = 0; s < nqs; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->p_full[s], 128);
      mbar_init(&bars->pv_done[s], 1);
      mbar_init(&bars->o_empty[s], 128);
    }
    mbar_init(&bars->kv_full, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) { tmem_alloc(&bars->tmem_base, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort;

  auto fail = [&]() {
    set_device_error(err, MSA_DEVERR_TIMEOUT);
    *abort_flag = 1;
  };

  if (warp == kIssuerWarp) {
    // ---------------------------------------------------------------- issuer
    if (lane == 0 && my_tiles > 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const uint32_t idS = idesc_bf16(128, kChunkKeys, 0, 0);
      const uint32_t idO = idesc_bf16(128, kD, 0, 1);
      int prev_seg = -1;
      uint32_t kvn = 0;
      bool ok = true;
      // Descriptor bases, computed once: an MMA k-step only adds a constant offset (in
      // 16-byte units) to the start-address field.
      // Q stages and K/V chunks are 32 KB apart: (2 * kTileBytes) >> 4 descriptor units.
      constexpr uint64_t kStep = (2 * kTileBytes) >> 4;
      const uint64_t qdesc0 = sdesc_sw128(smem_u32(Qs), 16, 1024);
      const uint64_t kdesc0 = sdesc_sw128(smem_u32(Ks), 16, 1024);
      const uint64_t vdesc0 = sdesc_sw128(smem_u32(Vs), kTileBytes, 1024);
      // QK of tile m, chunk c, into S_X
      auto issue_qk = [&](int m, int c) -> bool {
        const int X = m & 1;
        const int qs = m % nqs;
        // S_X is overwritten while an earlier PV may still be reading P_X from it: the
        // MMAs of this thread execute in issue order, so no completion wait is needed.
        if (c == 0 && !mbar_wait(&bars->q_full[qs], (m / nqs) & 1)) return false;
        tc_fence_after();
        const uint64_t qd = qdesc0 + (uint64_t)qs * kStep, kd = kdesc0 + (uint64_t)c * kStep;
        const uint32_t dt = tmem + X * 128;
#pragma unroll
        for (int s = 0; s < kD / 16; ++s) {
          const uint64_t off = (uint64_t)((s >> 2) * (kTileBytes >> 4) + (s & 3) * 2);
          umma_ss(dt, qd + off, kd + off, idS, s > 0);
        }
        umma_commit(&bars->s_full[X]);
        if (c == nch - 1) umma_commit(&bars->q_empty[qs]);
        return true;
      };
      // PV of tile m, chunk c, into O_X (P read from TMEM over S_X)
      auto issue_pv = [&](int m, int c) -> bool {
        const int X = m & 1;
        if (!mbar_wait(&bars->p_full[X], chunk_phase(m, c, nch))) return false;
        if (c == 0 && m >= 2 && !mbar_wait(&bars->o_empty[X], ((m >> 1) - 1) & 1)) return false;
        tc_fence_after();
        const uint64_t vd = vdesc0 + (uint64_t)c * kStep;
        const uint32_t dt = tmem + 256 + X * 128, at = tmem + X * 128;
#pragma unroll
        for (int s = 0; s < kChunkKeys / 16; ++s)
          umma_ts(dt, at + s * 8, vd + (uint64_t)(s * (2048 >> 4)), idO, (c > 0 || s > 0) ? 1u : 0u);
        umma_commit(&bars->pv_done[X]);
        return true;
      };
      // Runs of consecutive tiles share one segment's K/V.  Inside a run the tiles are
      // two streams (tiles n, n+2, ... and n+1, n+3, ...), issued alternately one unit
      // at a time, a unit being [wait P] PV(m, c) followed by the stream's next QK: chunk
      // c+1 of m, or chunk 0 of m+2.  So one tile's MMAs run while the other tile's
      // warpgroup does its softmax (the two are half a unit apart).
      auto rec_x = [&](int m) -> int { return m < my_tiles ? tiles[tile_lo + m].x : -1; };
      int n = 0, last_pv = -1;
      while (n < my_tiles && ok) {
        if (*abort_flag) break;
        const int4 tl = tiles[tile_lo + n];
        // the stream whose turn it is (a) and the other (b): tile, next chunk, segment of
        // the stream's next tile, still active
        int ma = n, ca = 0, xa = rec_x(n + 2);
        bool aa = true;
        int mb = n + 1, cb = 0, xb = -1;
        bool ab = rec_x(n + 1) == tl.x;
        if (ab) xb = rec_x(n + 3);
        if (tl.x != prev_seg) {
          // every MMA of earlier tiles must be done before K/V are overwritten
          if (last_pv >= 0 &&
              !mbar_wait(&bars->pv_done[last_pv & 1], chunk_phase(last_pv, nch - 1, nch))) {
            ok = false;
            break;
          }
          const TileId id = decode_tile(tl, g);
          const int y0 = (int)((int64_t)id.b * g.S + (int64_t)id.j * g.block +
                               (int64_t)id.sub * kSegKeys);
          const int64_t gg = id.gg;
          mbar_arrive_expect_tx(&bars->kv_full, (uint32_t)(nch * 4 * kTileBytes));
          for (int cc = 0; cc < nch; ++cc)
            for (int hf = 0; hf < 2; ++hf) {
              const int x = (int)(gg * kD + hf * 64);
              tma_load_2d(Ks + (cc * 2 + hf) * kTileBytes, &tmK, &bars->kv_full, x,
                          y0 + cc * kChunkKeys);
              tma_load_2d(Vs + (cc * 2 + hf) * kTileBytes, &tmV, &bars->kv_full, x,
                          y0 + cc * kChunkKeys);
            }
          if (!mbar_wait(&bars->kv_full, kvn & 1)) { ok = false; break; }
          ++kvn;
          prev_seg = tl.x;
        }
        int end = ab ? n + 2 : n + 1;                    // one past the last tile started
        ok = issue_qk(ma, 0);
        if (ok && ab) ok = issue_qk(mb, 0);
        while (ok && (aa || ab)) {
          if (aa) {
            if (*abort_flag) { ok = false; break; }
            ok = issue_pv(ma, ca);
            last_pv = ma;
            if (!ok) break;
            if (ca + 1 < nch) {
              ++ca;
              ok = issue_qk(ma, ca);
            } else if (xa == tl.x) {                     // the stream's next tile, same K/V
              ma += 2;
              ca = 0;
              xa = rec_x(ma + 2);
              ok = issue_qk(ma, 0);
              end = ma + 1 > end ? ma + 1 : end;
            } else {
              aa = false;
            }
          }
          // the other stream's turn
          int t_m = ma, t_c = ca, t_x = xa;
          bool t_a = aa;
          ma = mb; ca = cb; xa = xb; aa = ab;
          mb = t_m; cb = t_c; xb = t_x; ab = t_a;
        }
        n = end;
      }
      if (!ok) fail();
    }
  } else if (warp == kGatherWarp) {
    // ---------------------------------------------------------------- Q gather
    // Tensor-map copies: viewed as [b*S*hq, 128], a token's G query heads of group gg are
    // G consecutive rows, so each (token, 64-dim half) is one box of G rows, landing at
    // tile rows [G*i, G*i+G) in the 128-byte-swizzled layout the MMA reads.  Each lane
    // copies its own tokens; one arrive with the tile's byte count publishes the stage.
    // Tile n+1's token ids and tile n+2's record are loaded while tile n's copies go out.
    constexpr int kTok = kRowsT / G;                     // tokens per tile
    constexpr int kPerLane = (kTok + 31) / 32;
    if (lane == 0 && my_tiles > 0) prefetch_tmap(&tmQ);
    int4 tl_n = my_tiles > 0 ? tiles[tile_lo] : make_int4(0, 0, 0, 0);
    int4 tl_n1 = my_tiles > 1 ? tiles[tile_lo + 1] : make_int4(0, 0, 0, 0);
    int ent_n[kPerLane];
#pragma unroll
    for (int u = 0; u < kPerLane; ++u) {
      const int i = lane + u * 32;
      ent_n[u] = (my_tiles > 0 && i < kTok && i < tl_n.z) ? entries[tl_n.y + i] : -1;
    }
    int issued = 0;                                      // tiles whose copies went out
    for (int n = 0; n < my_tiles; ++n) {
      const int st = n % nqs;
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      if (n >= nqs && !mbar_wait_warp(&bars->q_empty[st], ((n / nqs) - 1) & 1)) {
        if (lane == 0) fail();
        break;
      }
      const int4 tl = tl_n;
      int ent[kPerLane];
      int n_valid = 0;
#pragma unroll
      for (int u = 0; u < kPerLane; ++u) {
        ent[u] = ent_n[u];
        n_valid += __popc(__ballot_sync(0xffffffffu, ent[u] >= 0));
      }
      if (n + 1 < my_tiles) {                            // tile n+1's token ids
#pragma unroll
        for (int u = 0; u < kPerLane; ++u) {
          const int i = lane + u * 32;
          ent_n[u] = (i < kTok && i < tl_n1.z) ? entries[tl_n1.y + i] : -1;
        }
        tl_n = tl_n1;
      }
      if (n + 2 < my_tiles) tl_n1 = tiles[tile_lo + n + 2];   // tile n+2's record
      if (lane == 0) mbar_arrive_expect_tx(&bars->q_full[st], (uint32_t)(n_valid * G * kD * 2));
      __syncwarp();
      const int b = tl.w / g.hkv, gg = tl.w - b * g.hkv;
      unsigned char* qb = Qs + st * 2 * kTileBytes;
#pragma unroll
      for (int u = 0; u < kPerLane; ++u) {
        if (ent[u] < 0) continue;
        const int i = lane + u * 32;
        const int y = (int)(((int64_t)b * g.S + (ent[u] >> 6)) * g.hq + gg * G);
        tma_load_2d(qb + i * G * 128, &tmQ, &bars->q_full[st], 0, y);
        tma_load_2d(qb + kTileBytes + i * G * 128, &tmQ, &bars->q_full[st], 64, y);
      }
      issued = n + 1;
    }
    // no copy may still be landing when the CTA exits (normally all were consumed)
    for (int m = issued > nqs ? issued - nqs : 0; m < issued; ++m)
      if (!mbar_wait_warp(&bars->q_full[m % nqs], (m / nqs) & 1)) break;
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    const int X = warp >> 2;                             // this warpgroup's tile parity
    const int r = tid & 127;                             // TMEM lane = tile row
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t sX = lane_base + X * 128, oX = lane_base + 256 + X * 128;
    const int tok = r / G, h = r % G;
    const float c2 = g.scale_log2;
    int4 tl_next = X < my_tiles ? tiles[tile_lo + X] : make_int4(0, 0, 0, 0);
    int e_next = (X < my_tiles && tok < tl_next.z) ? entries[tl_next.y + tok] : -1;
    for (int n = X; n < my_tiles; n += 2) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      const int4 tl = tl_next;
      const int ent = e_next;
      if (n + 2 < my_tiles) {                            // this warpgroup's next tile
        tl_next = tiles[tile_lo + n + 2];
        e_next = tok < tl_next.z ? entries[tl_next.y + tok] : -1;
      }
      const TileId id = decode_tile(tl, g);
      const int sub = id.sub;
      const int64_t j = id.j, gg = id.gg, b = id.b;
      const bool valid = ent >= 0;
      const int64_t t = valid ? (ent >> 6) : 0;
      const int pslot = valid ? (ent & 63) : 0;
      const int64_t own = (int)t / (int)g.block;
      const int64_t kbase = j * g.block + (int64_t)sub * kSegKeys;
      int64_t khi = (j == own) ? t + 1 : j * g.block + g.block;
      const int64_t seg_end = j * g.block + min((int64_t)(sub + 1) * kSegKeys, g.block);
      khi = min(min(khi, seg_end), g.S);
      float mref = -CUDART_INF_F;      // exponent reference (scaled, base 2)
      float l = 0.f;
      bool ok = true;
      for (int c = 0; c < nch; ++c) {
        const int64_t rem = khi - (kbase + (int64_t)c * kChunkKeys);
        const int lim = valid ? (int)max((int64_t)0, min((int64_t)kChunkKeys, rem)) : 0;
        const uint32_t ph = chunk_phase(n, c, nch);
        if (!mbar_wait_warp(&bars->s_full[X], ph)) { ok = false; break; }
        tc_fence_after();
        const bool full = __all_sync(0xffffffffu, lim == kChunkKeys);
        // One pass over S in two halves of 64 columns.  Each half's max is taken from the
        // registers just loaded; the exponent reference mref only moves when a half's max
        // exceeds it by more than 2^8 (always for the first half of a row's first chunk),
        // and then O, l, and the P already made for this chunk are rescaled.
        float sum = 0.f;
        bool o_ready = c == 0;                           // O holds nothing to rescale yet
#pragma unroll
        for (int hq2 = 0; hq2 < 2; ++hq2) {
          uint32_t sv[2][32];
          tmem_ld32(sX + hq2 * 64, sv[0]);
          tmem_ld32(sX + hq2 * 64 + 32, sv[1]);
          tmem_ld_wait();
          float mx = -CUDART_INF_F;
          if (full) {
            // eight independent chains of three-input maxima
            float m8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const uint32_t* v = &sv[i >> 2][(i & 3) * 8];
              float m = fmax3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]));
              m = fmax3(m, __uint_as_float(v[3]), __uint_as_float(v[4]));
              m = fmax3(m, __uint_as_float(v[5]), __uint_as_float(v[6]));
              m8[i] = fmaxf(m, __uint_as_float(v[7]));
            }
            mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]),
                       fmaxf(m8[6], m8[7]));
          } else {
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int qd = hq2 * 2 + u;
#pragma unroll
              for (int k = 0; k < 32; ++k)
                if (qd * 32 + k < lim) mx = fmaxf(mx, __uint_as_float(sv[u][k]));
            }
          }
          const float mc = lim > hq2 * 64 ? mx * c2 : -CUDART_INF_F;
          const bool need = mc > mref + kRescaleLog2;
          if (__any_sync(0xffffffffu, need)) {
            const float f = need ? fast_exp2(mref - mc) : 1.f;
            if (!o_ready) {
              // O must hold every earlier chunk before it is rescaled in TMEM
              if (!mbar_wait_warp(&bars->pv_done[X], chunk_phase(n, c - 1, nch))) {
                ok = false;
                break;
              }
              tc_fence_after();
              o_ready = true;
            }
            // (rare) rescale in 16-column pieces, keeping S of this half in registers
            if (c > 0) {
#pragma unroll 1
              for (int qd = 0; qd < 8; ++qd) {
                uint32_t ov[16];
                tmem_ld16(oX + qd * 16, ov);
                tmem_ld_wait();
#pragma unroll
                for (int k = 0; k < 16; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * f);
                tmem_st16(oX + qd * 16, ov);
              }
              tmem_st_wait();
            }
            if (hq2 == 1) {                             // this chunk's first half of P
              tmem_st_wait();
#pragma unroll 1
              for (int qd = 0; qd < 2; ++qd) {
                uint32_t pv[16];
                tmem_ld16(sX + qd * 16, pv);
                tmem_ld_wait();
#pragma unroll
                for (int k = 0; k < 16; ++k)
                  pv[k] = pack_bf16x2(bf16lo_to_f32(pv[k]) * f, bf16hi_to_f32(pv[k]) * f);
                tmem_st16(sX + qd * 16, pv);
              }
            }
            l *= f;
            sum *= f;
            if (need) mref = mc;
          }
          const float mb = mref > -CUDART_INF_F ? mref : 0.f;
          uint32_t pk[32];
          // Two lanes per instruction.  The pairs MSA_POLY_PAIRS marks take their
          // exponentials on the FMA pipe, the rest on the MUFU unit; columns past lim
          // (ragged or causal rows) become 0.  The arithmetic of a column does not depend
          // on whether other rows of the warp are ragged.
          float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
          for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int k = 0; k < 32; k += 2) {
              float x0, x1, p0, p1;
              ffma2(x0, x1, __uint_as_float(sv[u][k]), __uint_as_float(sv[u][k + 1]), c2, c2,
                    -mb, -mb);
              if ((MSA_POLY_PAIRS >> ((k / 2) & 7)) & 1) {
                poly_exp2x2(x0, x1, p0, p1);
              } else {
                p0 = fast_exp2(x0);
                p1 = fast_exp2(x1);
              }
              if (!full) {
                const int kk = (hq2 * 2 + u) * 32 + k;
                p0 = kk < lim ? p0 : 0.f;
                p1 = kk + 1 < lim ? p1 : 0.f;
              }
              if (u == 0) fadd2(a0, a1, a0, a1, p0, p1);
              else fadd2(b0, b1, b0, b1, p0, p1);
              pk[u * 16 + k / 2] = pack_bf16x2(p0, p1);
            }
          sum += (a0 + a1) + (b0 + b1);
          // P of this half over S columns already consumed
          tmem_st32(sX + hq2 * 32, pk);
        }
        if (!ok) break;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars->p_full[X]);
        l += sum;
      }
      if (!ok || !mbar_wait_warp(&bars->pv_done[X], chunk_phase(n, nch - 1, nch))) {
        fail();
        break;
      }
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const int64_t prow = (b * g.hkv + gg) * g.slab + (t - g.t_base);   // partial row of the slab
      __nv_bfloat16* dst = po + ((prow * g.kslots + pslot) * G + h) * kD;
      // O in two halves of 64 columns, two TMEM loads in flight per wait
#pragma unroll 1
      for (int q2 = 0; q2 < 2; ++q2) {
        uint32_t ov[2][32];
        tmem_ld32(oX + q2 * 64, ov[0]);
        tmem_ld32(oX + q2 * 64 + 32, ov[1]);
        tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          uint32_t ob[16];
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            float y0, y1;
            fmul2(y0, y1, __uint_as_float(ov[u][k]), __uint_as_float(ov[u][k + 1]), inv, inv);
            ob[k / 2] = pack_bf16x2(y0, y1);
          }
          if (valid) {
            st_global_v8(dst + (q2 * 2 + u) * 32, ob);
            st_global_v8(dst + (q2 * 2 + u) * 32 + 16, ob + 8);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->o_empty[X]);
      if (valid)
        plse[(prow * g.kslots + pslot) * G + h] =
            l > 0.f ? (mref + log2f(l)) * kLn2 : -CUDART_INF_F;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ merge partials
// One row = (sequence, group, token); G*8 threads per row, 16 output elements (32 bytes)
// each.  One pass over the row's partials with a running max, kMergeBatch loads in flight
// per thread.
constexpr int kMergeBatch = 4;   // 8 measured 2% slower at 1M
__device__ __forceinline__ void ld_global_nc_v8(const void* p, uint32_t* r) {
  asm volatile("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "l"(p));
}

template <int G>
__global__ void __launch_bounds__(128)
merge_partials_kernel(const int32_t* __restrict__ idx, const __nv_bfloat16* __restrict__ po,
                      const float* __restrict__ plse, __nv_bfloat16* __restrict__ o,
                      float* __restrict__ lse, Geom g, int64_t n_rows) {
  constexpr int TPR = G * 8;
  constexpr int RPC = 128 / TPR;
  const int64_t row = (int64_t)blockIdx.x * RPC + threadIdx.x / TPR;
  if (row >= n_rows) return;
  const int lt = threadIdx.x % TPR;
  const int h = lt / 8;
  // partial row `row` of the slab = (sequence*hkv + group, token t_base + row % slab)
  const int64_t bg = row / g.slab;
  const int t = (int)(g.t_base + row % g.slab);
  if (t >= g.t_end) return;
  const int64_t gg = bg % g.hkv, b = bg / g.hkv;
  const int own = t / (int)g.block;
  const int32_t* irow = idx + (bg * g.S + t) * g.topk;
  const float* lrow = plse + row * g.kslots * G;
  const __nv_bfloat16* prow = po + row * g.kslots * G * kD + lt * 16;
  float mx = -CUDART_INF_F, den = 0.f;
  float acc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] = 0.f;
  int ps_list[kMergeBatch];
  int np = 0;
  auto flush = [&]() {
    float lv[kMergeBatch];
    uint32_t raw[kMergeBatch][8];
#pragma unroll
    for (int u = 0; u < kMergeBatch; ++u)
      if (u < np) {
        lv[u] = lrow[ps_list[u] * G + h];
        ld_global_nc_v8(prow + (int64_t)ps_list[u] * G * kD, raw[u]);
      }
#pragma unroll
    for (int u = 0; u < kMergeBatch; ++u) {
      if (u >= np || !(lv[u] > -CUDART_INF_F)) continue;
      const float mn = fmaxf(mx, lv[u]);
      const float sc = exp2f((mx - mn) * kLog2e);
      const float wgt = exp2f((lv[u] - mn) * kLog2e);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        acc[2 * e] = fmaf(wgt, bf16lo_to_f32(raw[u][e]), acc[2 * e] * sc);
        acc[2 * e + 1] = fmaf(wgt, bf16hi_to_f32(raw[u][e]), acc[2 * e + 1] * sc);
      }
      den = den * sc + wgt;
      mx = mn;
    }
    np = 0;
  };
  for (int sl = 0; sl < g.topk; ++sl) {
    const int j = irow[sl];
    if (j < 0 || j >= g.nb || j > own) continue;
    for (int sub = 0; sub < g.nsub; ++sub) {
      if (!sub_has_keys32(j, own, t, sub, g)) continue;
      ps_list[np++] = sl * g.nsub + sub;
      if (np == kMergeBatch) flush();
    }
  }
  if (np > 0) flush();
  const float inv = den > 0.f ? 1.f / den : 0.f;
  uint32_t out[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) out[e] = pack_bf16x2(acc[2 * e] * inv, acc[2 * e + 1] * inv);
  __nv_bfloat16* dst = o + ((b * g.S + t) * g.hq + gg * G) * kD + lt * 16;
  if ((reinterpret_cast<uintptr_t>(o) & 31) == 0) {   // the ABI only promises 16 bytes
    st_global_v8(dst, out);
  } else {
    reinterpret_cast<uint4*>(dst)[0] = make_uint4(out[0], out[1], out[2], out[3]);
    reinterpret_cast<uint4*>(dst)[1] = make_uint4(out[4], out[5], out[6], out[7]);
  }
  if (lse != nullptr && (lt % 8) == 0)
    lse[(b * g.hq + gg * G + h) * g.S + t] = den > 0.f ? mx + logf(den) : -CUDART_INF_F;
}

// ------------------------------------------------------------------ host side
struct WsLayout {
  size_t counts, seg_off, cursor, tile_off, n_tiles, entries, tiles, po, plse, total;
};

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

Geom make_geom(const Shape& s) {
  Geom g{};
  g.S = s.seq; g.nb = s.nb; g.block = s.block;
  g.hq = (int)s.hq; g.hkv = (int)s.hkv; g.G = (int)(s.hq / s.hkv); g.topk = (int)s.topk;
  g.nsub = (int)((s.block + kSegKeys - 1) / kSegKeys);
  g.kslots = g.topk * g.nsub;
  g.tpt = kRowsT / g.G;
  g.nch = (int)(((s.block < kSegKeys ? s.block : (int64_t)kSegKeys) + kChunkKeys - 1) / kChunkKeys);
  g.nseg = s.batch * s.hkv * s.nb * g.nsub;
  g.scale_log2 = s.scale * kLog2e;
  g.t_base = 0; g.t_end = s.seq; g.slab = s.seq;
  return g;
}

// Workspace of one call processing `slab` tokens of every (sequence, group) at a time: the
// per-segment index of the whole call, the entries and tiles of one slab, and the
// slab's partials (which dominate: kslots x G x 256 B + 4 B per (token, group)).
WsLayout layout_for(const Shape& s, int64_t slab) {
  const Geom g = make_geom(s);
  const int64_t n_entries = s.batch * s.hkv * slab * s.topk * g.nsub;
  const int64_t n_tiles_max = n_entries / g.tpt + g.nseg + 1;
  const int64_t rows = s.batch * s.hkv * slab;
  WsLayout L{};
  size_t o = 0;
  L.counts = o;   o += up256(g.nseg * 4);
  L.seg_off = o;  o += up256((g.nseg + 1) * 4);
  L.cursor = o;   o += up256(g.nseg * 4);
  L.tile_off = o; o += up256((g.nseg + 1) * 4);
  L.n_tiles = o;  o += 256;
  L.entries = o;  o += up256(n_entries * 4);
  L.tiles = o;    o += up256(n_tiles_max * 16);
  L.po = o;       o += up256((size_t)rows * g.kslots * g.G * kD * 2);
  L.plse = o;     o += up256((size_t)rows * g.kslots * g.G * 4);
  L.total = o;
  return L;
}

// Slabs are whole multiples of the inversion's token range (or the whole sequence).
constexpr size_t kSlabBudget = (size_t)32 << 30;   // recommended workspace: <= 32 GiB of slab
int64_t min_slab(const Shape& s) { return s.seq < kInvTokens ? s.seq : kInvTokens; }
int64_t slab_for(const Shape& s, size_t bytes) {
  if (layout_for(s, s.seq).total <= bytes) return s.seq;
  int64_t lo = 1, hi = s.seq / kInvTokens;         // in units of kInvTokens
  if (hi < 1) return s.seq;
  while (lo < hi) {                                // largest fitting multiple
    const int64_t mid = (lo + hi + 1) / 2;
    if (layout_for(s, mid * kInvTokens).total <= bytes) lo = mid; else hi = mid - 1;
  }
  // same number of slabs, evened out (never larger than the largest that fits)
  const int64_t units = (s.seq + kInvTokens - 1) / kInvTokens;
  const int64_t n_slabs = (units + lo - 1) / lo;
  return (units + n_slabs - 1) / n_slabs * kInvTokens;
}

template <int G>
cudaError_t run_tc(const Shape& s, const Geom& g, const CUtensorMap& mk, const CUtensorMap& mv,
                   const CUtensorMap& mq, const int32_t* idx, void* o, float* lse, char* ws,
                   const WsLayout& L, int* err, cudaStream_t st) {
  const size_t smem = 1024 + (size_t)q_stages(g.nch) * 2 * kTileBytes +
                      (size_t)g.nch * 4 * kTileBytes + sizeof(Bars);
  cudaError_t e = cudaFuncSetAttribute(attn_tiles_kernel<G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  attn_tiles_kernel<G><<<sm_count(), kThreads3, smem, st>>>(
      mk, mv, mq, (const int4*)(ws + L.tiles), (const int*)(ws + L.n_tiles),
      (const int*)(ws + L.entries), (__nv_bfloat16*)(ws + L.po), (float*)(ws + L.plse), err, g);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t rows = s.batch * s.hkv * g.slab;
  const int rpc = 128 / (G * 8);
  merge_partials_kernel<G><<<(unsigned)((rows + rpc - 1) / rpc), 128, 0, st>>>(
      idx, (const __nv_bfloat16*)(ws + L.po), (const float*)(ws + L.plse), (__nv_bfloat16*)o,
      lse, g, rows);
  return cudaGetLastError();
}

}  // namespace

bool tc_attn_supported(const Shape& s) {
  if (s.dtype != MSA_BF16 || s.d != kD) return false;
  if (s.block % kChunkKeys != 0) return false;
  if (s.block > kSegKeys && s.block % kSegKeys != 0) return false;
  const int64_t G = s.hq / s.hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return false;
  const int64_t nsub = (s.block + kSegKeys - 1) / kSegKeys;
  if (s.topk * nsub > 64) return false;                       // pslot fits 6 bits
  if (s.seq >= ((int64_t)1 << 25)) return false;              // token fits 25 bits
  if (s.batch * s.seq * s.hq >= ((int64_t)1 << 31)) return false;   // q row fits a map coordinate
  if (s.batch * s.hkv * s.seq * s.topk * nsub >= ((int64_t)1 << 31)) return false;
  if (s.batch * s.seq >= ((int64_t)1 << 31)) return false;    // TMA row coordinate
  if (s.nb * nsub > 48 * 1024) return false;                  // inversion histogram in smem
  return true;
}

size_t tc_attn_ws_bytes(const Shape& s) {
  return layout_for(s, slab_for(s, kSlabBudget)).total;
}
size_t tc_attn_ws_min_bytes(const Shape& s) { return layout_for(s, min_slab(s)).total; }
int64_t tc_attn_slab_tokens(const Shape& s, size_t ws_body_bytes) {
  const int64_t slab = slab_for(s, ws_body_bytes);
  return layout_for(s, slab).total <= ws_body_bytes ? (slab < s.seq ? slab : s.seq) : 0;
}

cudaError_t launch_attn_prefill_tc(const Shape& s, const void* q, const void* k, const void* v,
                                   const int32_t* idx, void* o, float* lse, void* ws_body,
                                   size_t ws_body_bytes, int* err, cudaStream_t st) {
  Geom g = make_geom(s);
  const int64_t slab = slab_for(s, ws_body_bytes);
  const WsLayout L = layout_for(s, slab);
  if (L.total > ws_body_bytes) return cudaErrorInvalidValue;
  g.slab = slab;
  char* ws = reinterpret_cast<char*>(ws_body);
  CUtensorMap mk, mv, mq;
  if (!make_bf16_2d_map(&mk, k, s.batch * s.seq, s.hkv * kD, 128) ||
      !make_bf16_2d_map(&mv, v, s.batch * s.seq, s.hkv * kD, 128) ||
      !make_bf16_2d_map(&mq, q, s.batch * s.seq * s.hq, kD, g.G))   // G heads per box
    return cudaErrorInvalidValue;
  const size_t hsmem = (size_t)g.nb * g.nsub * sizeof(int);
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(invert_hist_kernel<false>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hsmem)) !=
          cudaSuccess ||
      (e = cudaFuncSetAttribute(invert_hist_kernel<true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hsmem)) !=
          cudaSuccess)
    return e;
  // one pass per token slab: invert its selections, attend its tiles, merge its rows
  for (int64_t t0 = 0; t0 < s.seq; t0 += slab) {
    g.t_base = t0;
    g.t_end = t0 + slab < s.seq ? t0 + slab : s.seq;
    if ((e = cudaMemsetAsync(ws + L.counts, 0, g.nseg * 4, st)) != cudaSuccess) return e;
    const int64_t n_sel = s.batch * s.hkv * (g.t_end - t0) * s.topk;
    const dim3 hgrid((unsigned)((g.t_end - t0 + kInvTokens - 1) / kInvTokens),
                     (unsigned)(s.batch * s.hkv));
    invert_hist_kernel<false><<<hgrid, kInvThreads, hsmem, st>>>(
        idx, (int*)(ws + L.counts), nullptr, nullptr, err, g);
    invert_scan_kernel<<<1, 1024, 0, st>>>((const int*)(ws + L.counts), (int*)(ws + L.seg_off),
                                           (int*)(ws + L.cursor), (int*)(ws + L.tile_off),
                                           (int*)(ws + L.n_tiles), g.nseg, g.tpt);
    invert_hist_kernel<true><<<hgrid, kInvThreads, hsmem, st>>>(
        idx, nullptr, (int*)(ws + L.cursor), (int*)(ws + L.entries), err, g);
    const int64_t n_tiles_max = n_sel * g.nsub / g.tpt + g.nseg + 1;
    tile_table_kernel<<<(unsigned)((n_tiles_max + 255) / 256), 256, 0, st>>>(
        (const int*)(ws + L.counts), (const int*)(ws + L.seg_off), (const int*)(ws + L.tile_off),
        (const int*)(ws + L.n_tiles), (int4*)(ws + L.tiles), g.nseg, g.tpt,
        (int64_t)g.nb * g.nsub);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    switch (g.G) {
      case 1: e = run_tc<1>(s, g, mk, mv, mq, idx, o, lse, ws, L, err, st); break;
      case 2: e = run_tc<2>(s, g, mk, mv, mq, idx, o, lse, ws, L, err, st); break;
      case 4: e = run_tc<4>(s, g, mk, mv, mq, idx, o, lse, ws, L, err, st); break;
      default: e = run_tc<8>(s, g, mk, mv, mq, idx, o, lse, ws, L, err, st); break;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace msa
