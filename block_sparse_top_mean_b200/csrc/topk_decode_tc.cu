// Steps 2+3 for decode against a memory bank, on the tensor cores (bf16 queries, d = 128).
//
// The bank's pooled keys are stored as bf16 hi/lo planes (hi = bf16(kbar), lo =
// bf16(kbar - hi)), an offline encoding of the routing keys.  Each CTA streams a
// contiguous range of (group, 128-block chunk) units of the bank through a TMA ring and
// scores them against up to 64 queries:
//     S^T = Khi Qhi^T + Khi Qlo^T + Klo Qhi^T     (M = 128 blocks, N = 64 queries, K = 16)
// where Q is the group-summed query (fp32 sum over the group's heads) split the same
// way; the three terms reproduce the fp32 dot product to ~2^-17 relative.  Scores land in
// one of four TMEM accumulators, so the MMAs of later chunks overlap the filtering.
//
// Selection, exact under (score desc, block index asc):
//   - Eight epilogue warps read the accumulator: warp w holds TMEM lanes (blocks)
//     32*(w%4).. and the 32 queries 32*(w/4)...  Each thread tests its block's 32 scores
//     against T[n], the n-th query's current 32nd best score (shared memory), into a
//     32-bit pass mask; a warp OR of the masks finds the queries with any pass, and
//     only those are balloted and appended, as (score, block) keys, to the query's
//     pending list (one shared-memory atomic per warp and query).
//   - Each query's running top-32 lives in the registers of its owner warp (lane e
//     holds rank e; warp w owns queries w + 8 i).  After each chunk, owners whose
//     queries hold 32 or more pending keys merge the pending keys of all 8 owned queries
//     at once (a bitonic sort of each batch, the max against the reversed list, a
//     bitonic merge; the 8 independent networks overlap their latencies) and republish
//     T.  Dropping a score < T is safe: the 32 listed blocks all score at least T.
//   - At the end of a group's range the owner flushes its lists, sorted, to the candidate
//     array; topk_decode_merge_kernel merges the lists of the CTAs that shared the group
//     and writes the selection ascending.
// Long banks first run a sample pass over every 8th chunk that only records, per query,
// the maximum score of each 32-block group; the 32nd largest of those maxima (32
// different blocks reach it) seeds T for the full scan, so few blocks get appended.
// Keys are 64-bit: order-preserving bits of the score above the complement of the block
// index, so a larger key is a better block; key 0 is "empty".
#include <cudaTypedefs.h>
#include <math_constants.h>

#include "common.cuh"
#include "decode_keys.cuh"
#include "sm100.cuh"

namespace msa {
namespace {

using namespace sm100;
using namespace keys;

constexpr int kD = 128;
constexpr int kM = 128;                   // bank blocks per chunk (MMA M, TMEM lanes)
constexpr int kN = 64;                    // queries per CTA (MMA N)
constexpr int kStages = 3;                // TMA ring of half-chunks (64 dims, hi + lo)
constexpr int kStagesMax = 11;            // the deepest ring (hi-only filter scan)
constexpr int kAcc = 8;                   // TMEM accumulators of kN columns (all 512)
constexpr int kList = 32;                 // running list length per query (>= topk)
constexpr int kCand = 64;                 // candidates per query of the hi-plane scan
constexpr int kPend = 160;                // pending keys per query: < 32 kept + 128 new
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kThreads = kEpiThreads + 64;   // + TMA producer warp, MMA issuer warp
constexpr int kOwned = kN / kEpiWarps;    // queries per owner warp
constexpr uint32_t kPlane = 16384;        // 128 rows x 128 B: one plane of a half-chunk
constexpr uint32_t kStageBytes = 2 * kPlane;
constexpr uint32_t kQHalf = 8192;         // 64 rows x 128 B: 64 dims of one query plane
constexpr uint32_t kQBytes = 4 * kQHalf;  // per 64-dim half: hi rows, then lo rows

struct __align__(8) DBars {
  uint64_t full[kStagesMax], empty[kStagesMax], acc_full[kAcc], acc_empty[kAcc], q_full;
  uint32_t tmem_base;
  int abort;
};

struct DecGeom {
  int64_t nb;        // bank blocks
  int64_t n_query;
  int64_t nch;       // units (chunks visited) per group in this pass
  int64_t stride;    // chunk index of unit c is c * stride (1, or the sample stride)
  int64_t per;       // units (group, chunk) per CTA along x
  int64_t nq_pad;    // query tiles * kN
  int64_t nch_full;  // 128-block chunks per group of the whole bank (encoded-plane stride)
  const int* run_if;     // when given, the kernels exit at once unless *run_if != 0
  int* seg_count;        // filter mode: keys per segment [hkv][CTA slot][query] (may
                         // exceed kSegCap: the segment overflowed)
  int hq, hkv, G, topk, ns_max, ncta_x;
};


// Scan modes: bit 0 = sample pass (group maxima instead of lists); bit 1 = hi plane only
// (S^T = Khi Qhi^T + Khi Qlo^T, kCand-key lists, a candidate pre-selection); bit 2 =
// filter: every (query, block) score at or above the query's starting bound (tinit,
// required) is stored to the row's segment for this CTA in global memory, and no lists
// are kept; the epilogue warps then never wait for one another, and the shared memory
// of the pending lists goes to a deeper TMA ring.
constexpr int kModeSample = 1;
constexpr int kModeHi = 2;
constexpr int kModeFilter = 4;
constexpr int kSegCap = 128;              // filter keys per (row, CTA) segment
constexpr int kFilterCap = 1024;          // filter keys per row the selection takes
constexpr int kMaxSegments = 256;         // CTAs that can share a group (>= SM count)

// The TMA ring and shared-memory layout of a mode: [Q planes][ring][pending lists, list
// modes only][counts][bounds][barriers].
__host__ __device__ constexpr bool mode_hi(int m) { return (m & kModeHi) != 0; }
__host__ __device__ constexpr bool mode_filter(int m) { return (m & kModeFilter) != 0; }
__host__ __device__ constexpr int ring_stages(int m) {
  return mode_filter(m) ? (mode_hi(m) ? kStagesMax : 5) : (mode_hi(m) ? 2 * kStages : kStages);
}
__host__ __device__ constexpr uint32_t stage_bytes(int m) {
  return mode_hi(m) ? kPlane : kStageBytes;
}
__host__ __device__ constexpr size_t pend_bytes(int m) {
  return mode_filter(m) ? 0 : (size_t)kN * kPend * 8;
}
__host__ __device__ constexpr size_t smem_bytes(int m) {
  return 1024 + kQBytes + (size_t)ring_stages(m) * stage_bytes(m) + pend_bytes(m) +
         (size_t)kN * 8 + sizeof(DBars);
}
static_assert(smem_bytes(kModeFilter | kModeHi) <= 232448, "shared memory");
static_assert(smem_bytes(kModeFilter) <= 232448, "shared memory");
static_assert(smem_bytes(0) <= 232448, "shared memory");
static_assert(ring_stages(kModeFilter | kModeHi) <= kStagesMax, "barriers");

// Merges up to 32 pending keys of each of the warp's owned queries into their lists
// (warp-collective; the networks are independent, so their shuffles overlap).
// pend(i): pending keys of owned query i; c: pending counts (uniform, each < kPend);
// afterwards every count is max(c - 32, 0) and T holds the new 32nd best scores.
__device__ __forceinline__ void joint_drain(uint64_t (&y)[kOwned], float (&T)[kOwned],
                                            int (&c)[kOwned], uint64_t* pend, int warp,
                                            int lane) {
  // Stage loops stay rolled (the body already holds independent networks), which keeps
  // the epilogue small enough for the instruction cache.
  uint64_t x[kOwned];
#pragma unroll
  for (int i = 0; i < kOwned; ++i)
    x[i] = lane < c[i] ? pend[(size_t)(warp + kEpiWarps * i) * kPend + lane] : 0ull;
#pragma unroll 1
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll 1
    for (int j = k >> 1; j > 0; j >>= 1) {
      const bool take_max = ((lane & j) == 0) == ((lane & k) == 0);
#pragma unroll
      for (int i = 0; i < kOwned; ++i) {
        const uint64_t p = __shfl_xor_sync(0xffffffffu, x[i], j);
        x[i] = take_max ? umax64(x[i], p) : umin64(x[i], p);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kOwned; ++i) y[i] = umax64(y[i], __shfl_sync(0xffffffffu, x[i], 31 - lane));
#pragma unroll 1
  for (int j = 16; j > 0; j >>= 1) {
    const bool lower = (lane & j) == 0;
#pragma unroll
    for (int i = 0; i < kOwned; ++i) {
      const uint64_t p = __shfl_xor_sync(0xffffffffu, y[i], j);
      y[i] = lower ? umax64(y[i], p) : umin64(y[i], p);
    }
  }
  // keys beyond the first 32 move to the front (at most 127, in rounds of 32)
#pragma unroll
  for (int i = 0; i < kOwned; ++i) {
    uint64_t* pq = pend + (size_t)(warp + kEpiWarps * i) * kPend;
    const int rem = c[i] - 32;
    for (int o = 0; o < rem; o += 32) {
      uint64_t t = 0ull;
      if (o + lane < rem) t = pq[32 + o + lane];
      __syncwarp();
      if (o + lane < rem) pq[o + lane] = t;
      __syncwarp();
    }
    c[i] = rem > 0 ? rem : 0;
    // never below a starting bound the list has not reached yet
    T[i] = fmaxf(T[i], key_score(__shfl_sync(0xffffffffu, y[i], kList - 1)));
  }
}

// The group-summed query of the tile's queries for group gg, split into bf16 hi and lo
// planes (B operands, 128-byte swizzle); epilogue thread `tid` writes its share.
template <int G, int NT = kEpiThreads>
__device__ __forceinline__ void write_query_planes(unsigned char* QI,
                                                   const __nv_bfloat16* __restrict__ q,
                                                   int64_t qt, int nqv, int gg, int hq, int tid) {
#pragma unroll 1
  for (int e = tid; e < kN * 16; e += NT) {
    const int n = e >> 4, cc16 = e & 15, hf = cc16 >> 3, cc = cc16 & 7;
    float acc8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (n < nqv) {
      const __nv_bfloat16* qr = q + ((qt * kN + n) * (int64_t)hq + (int64_t)gg * G) * kD + cc16 * 8;
      uint4 raw[G];
#pragma unroll
      for (int h = 0; h < G; ++h) raw[h] = ldg16(qr + (int64_t)h * kD);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float f[8];
        Vec16<__nv_bfloat16>::unpack(raw[h], f);
#pragma unroll
        for (int k = 0; k < 8; ++k) acc8[k] += f[k];
      }
    }
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
      const uint32_t hp = pack_bf16x2(acc8[k], acc8[k + 1]);
      hw[k / 2] = hp;
      lw[k / 2] = pack_bf16x2(acc8[k] - bf16lo_to_f32(hp), acc8[k + 1] - bf16hi_to_f32(hp));
    }
    const uint32_t off = (uint32_t)n * 128u + ((uint32_t)(cc ^ (n & 7)) << 4);
    // half hf: the hi plane's 64 rows, then the lo plane's: one 128-row B operand
    *reinterpret_cast<uint4*>(QI + (2 * hf) * kQHalf + off) =
        make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4*>(QI + (2 * hf + 1) * kQHalf + off) =
        make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
}

// Bit n of the result: score v[n] reaches threshold t[n] (n < 32; t 16-byte aligned).
__device__ __forceinline__ uint32_t pass_mask(const uint32_t (&v)[32], const float* t) {
  uint32_t pm = 0u;
#pragma unroll
  for (int n4 = 0; n4 < 8; ++n4) {
    const float4 t4 = *reinterpret_cast<const float4*>(t + n4 * 4);
    pm |= (__uint_as_float(v[n4 * 4 + 0]) >= t4.x ? 1u : 0u) << (n4 * 4 + 0);
    pm |= (__uint_as_float(v[n4 * 4 + 1]) >= t4.y ? 1u : 0u) << (n4 * 4 + 1);
    pm |= (__uint_as_float(v[n4 * 4 + 2]) >= t4.z ? 1u : 0u) << (n4 * 4 + 2);
    pm |= (__uint_as_float(v[n4 * 4 + 3]) >= t4.w ? 1u : 0u) << (n4 * 4 + 3);
  }
  return pm;
}

// This thread's 32 scores of an accumulator (TMEM address `taddr`): HI = the two terms
// in columns c and c + 64, added in fp32.
template <bool HI>
__device__ __forceinline__ void load_scores(uint32_t taddr, uint32_t (&v)[32]) {
  tmem_ld32(taddr, v);
  if constexpr (HI) {
    uint32_t w[32];
    tmem_ld32(taddr + kN, w);
    tmem_ld_wait();
#pragma unroll
    for (int n = 0; n < 32; ++n)
      v[n] = __float_as_uint(__uint_as_float(v[n]) + __uint_as_float(w[n]));
  } else {
    tmem_ld_wait();
  }
}

// v[n] for a warp-uniform n (a select tree: no dynamic register indexing).
__device__ __forceinline__ uint32_t pick32(const uint32_t (&v)[32], int n) {
  uint32_t a[16], b[8], c[4], d[2];
#pragma unroll
  for (int i = 0; i < 16; ++i) a[i] = (n & 16) ? v[i + 16] : v[i];
#pragma unroll
  for (int i = 0; i < 8; ++i) b[i] = (n & 8) ? a[i + 8] : a[i];
#pragma unroll
  for (int i = 0; i < 4; ++i) c[i] = (n & 4) ? b[i + 4] : b[i];
#pragma unroll
  for (int i = 0; i < 2; ++i) d[i] = (n & 2) ? c[i + 2] : c[i];
  return (n & 1) ? d[1] : d[0];
}

// Transposes a warp's 32x32 bit matrix: lane l's bit n -> lane n's bit l.
__device__ __forceinline__ uint32_t transpose32(uint32_t m, int lane) {
#pragma unroll
  for (int sh = 16; sh > 0; sh >>= 1) {
    const uint32_t lo = sh == 16 ? 0x0000ffffu : sh == 8 ? 0x00ff00ffu
                      : sh == 4 ? 0x0f0f0f0fu : sh == 2 ? 0x33333333u : 0x55555555u;
    const uint32_t o = __shfl_xor_sync(0xffffffffu, m, sh);
    m = (lane & sh) ? ((m & ~lo) | ((o >> sh) & lo)) : ((m & lo) | ((o << sh) & ~lo));
  }
  return m;
}

// MODE & kModeSample: the sample pass.  Instead of candidate lists the epilogue writes,
// per query, the maximum score of every 32-block group (its order-preserving bits) to
// gmax [query][group][sampled group index].
// MODE & kModeHi: only the hi plane is streamed (half the bytes) and scored against the
// split query: the sample and filter passes of a certified selection.
template <int G, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
topk_decode_tc_kernel(const __grid_constant__ CUtensorMap tmHi,
                      const __grid_constant__ CUtensorMap tmLo,
                      const unsigned char* __restrict__ ktiles,
                      const __nv_bfloat16* __restrict__ q, const float* __restrict__ tinit,
                      uint64_t* __restrict__ cand, uint32_t* __restrict__ gmax, int* err,
                      DecGeom g) {
  constexpr bool GMAX = (MODE & kModeSample) != 0;
  constexpr bool HI = (MODE & kModeHi) != 0;
  constexpr bool FILTER = (MODE & kModeFilter) != 0;
  static_assert(!(GMAX && FILTER), "the sample pass keeps group maxima");
  static_assert(!HI || GMAX || FILTER, "the hi-plane scan has no list form");
  constexpr int NST = ring_stages(MODE);                  // ring stages
  // accumulators: 64 columns (the three-term score), or 128 in the hi-plane modes (the
  // two terms side by side); all 512 TMEM columns either way
  constexpr uint32_t ACOLS = HI ? 2 * kN : kN;
  constexpr int NACC = (int)((kAcc * kN) / ACOLS);
  constexpr uint32_t SB = stage_bytes(MODE);              // bytes per stage
  if (g.run_if != nullptr && *(volatile const int*)g.run_if == 0) return;
  const int64_t total = (int64_t)g.hkv * g.nch;
  const int64_t u0 = (int64_t)blockIdx.x * g.per;
  const int64_t u1 = u0 + g.per < total ? u0 + g.per : total;
  if (u0 >= u1) return;                          // no units (uniform for the CTA)

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* QI = base;                                   // query planes (B operand)
  unsigned char* KS = QI + kQBytes;                           // stages: hi plane, lo plane
  uint64_t* pend = reinterpret_cast<uint64_t*>(KS + (size_t)NST * SB);   // [kN][kPend], lists
  int* cnt = reinterpret_cast<int*>(KS + (size_t)NST * SB + pend_bytes(MODE));   // [kN]
  float* Ts = reinterpret_cast<float*>(cnt + kN);                             // [kN]
  DBars* bars = reinterpret_cast<DBars*>(Ts + kN);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int64_t qt = blockIdx.y;
  const int nqv = (int)(g.n_query - qt * kN < kN ? g.n_query - qt * kN : kN);

  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int a = 0; a < kAcc; ++a) {
      mbar_init(&bars->acc_full[a], 1);
      mbar_init(&bars->acc_empty[a], kEpiWarps);
    }
    mbar_init(&bars->q_full, kEpiThreads);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (tid < kN) { cnt[tid] = 0; Ts[tid] = -CUDART_INF_F; }
  if (warp == 0) { tmem_alloc(&bars->tmem_base, kAcc * kN); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort;
  auto fail = [&]() { set_device_error(err, MSA_DEVERR_TIMEOUT); *abort_flag = 1; };

  if (warp == kEpiWarps) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const bool tiled = ktiles != nullptr;
      if (!tiled) {
        prefetch_tmap(&tmHi);
        prefetch_tmap(&tmLo);
      }
      int64_t step = 0;
      for (int64_t u = u0; u < u1 && !*abort_flag; ++u) {
        const int gg = (int)(u / g.nch);
        const int64_t chunk = (u % g.nch) * g.stride;
        const int y = (int)(chunk * kM);
        for (int hf = 0; hf < 2; ++hf, ++step) {
          const int st = (int)(step % NST);
          if (step >= NST &&
              !mbar_wait(&bars->empty[st], (uint32_t)((step / NST) - 1) & 1)) {
            fail();
            break;
          }
          unsigned char* dst = KS + st * SB;
          mbar_arrive_expect_tx(&bars->full[st], SB);
          if (tiled) {
            // encoded planes: [plane][group][chunk][half] images of 16 KB each
            const size_t plane = (size_t)g.hkv * g.nch_full * 2 * kPlane;
            const size_t off = (((size_t)gg * g.nch_full + chunk) * 2 + hf) * kPlane;
            bulk_load(dst, ktiles + off, kPlane, &bars->full[st]);
            if (!HI) bulk_load(dst + kPlane, ktiles + plane + off, kPlane, &bars->full[st]);
          } else {
            const int x = gg * kD + hf * 64;
            tma_load_2d(dst, &tmHi, &bars->full[st], x, y);
            if (!HI) tma_load_2d(dst + kPlane, &tmLo, &bars->full[st], x, y);
          }
        }
      }
    }
  } else if (warp == kEpiWarps + 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kM, kN, 0, 0);
      constexpr uint32_t idesc_hl = idesc_bf16(kM, 2 * kN, 0, 0);   // hi and lo rows at once
      const uint64_t qd = sdesc_sw128(smem_u32(QI), 16, 1024);
      const uint64_t kd0 = sdesc_sw128(smem_u32(KS), 16, 1024);
      int64_t step = 0, tile = 0;
      uint32_t seg = 0;
      for (int64_t u = u0; u < u1 && !*abort_flag; ++u, ++tile) {
        if (u == u0 || u % g.nch == 0) {              // new group: fresh query planes
          if (!mbar_wait(&bars->q_full, seg & 1)) { fail(); break; }
          ++seg;
        }
        const int a = (int)(tile % NACC);
        if (tile >= NACC &&
            !mbar_wait(&bars->acc_empty[a], (uint32_t)((tile / NACC) - 1) & 1)) {
          fail();
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + a * ACOLS;
        bool ok = true;
        for (int hf = 0; hf < 2; ++hf, ++step) {
          const int st = (int)(step % NST);
          if (!mbar_wait(&bars->full[st], (uint32_t)(step / NST) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint64_t kh = kd0 + (uint64_t)((st * SB) >> 4);
          const uint64_t kl = kh + (kPlane >> 4);
          const uint64_t qh = qd + (uint64_t)((2 * hf * kQHalf) >> 4);
          const uint64_t ql = qd + (uint64_t)(((2 * hf + 1) * kQHalf) >> 4);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t o = (uint64_t)(ks * 2);   // 32 bytes per k-step, in 16-B units
            if (HI) {
              // columns [0, 64): Khi.Qhi, [64, 128): Khi.Qlo (the epilogue adds them)
              umma_ss(acc, kh + o, qh + o, idesc_hl, (hf | ks) ? 1u : 0u);
            } else {
              umma_ss(acc, kh + o, qh + o, idesc, (hf | ks) ? 1u : 0u);
              umma_ss(acc, kh + o, ql + o, idesc, 1u);
              umma_ss(acc, kl + o, qh + o, idesc, 1u);
            }
          }
          umma_commit(&bars->empty[st]);
        }
        if (!ok) { fail(); break; }
        umma_commit(&bars->acc_full[a]);
      }
    }
  } else if constexpr (FILTER) {
    // ------------------------------------------------------------ filter epilogue (0-7)
    // warp w: TMEM lanes (blocks) 32*(w%4).., queries 32*(w/4)..  Passing keys go to the
    // row's segment for this CTA in global memory (a shared-memory counter per query
    // hands out the slots); at the end of the group's range the counts are published.
    // The epilogue warps meet only at group boundaries.
    const int quarter = warp & 3, qh = warp >> 2;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16) + qh * 32;
    const int nq_here = nqv - qh * 32;           // valid queries of this warp's 32
    bool aborted = false;
    int64_t tile = 0;
    int64_t u = u0;
    while (u < u1) {
      const int gg = (int)(u / g.nch);
      const int64_t ue = ((int64_t)gg + 1) * g.nch < u1 ? ((int64_t)gg + 1) * g.nch : u1;
      const int64_t nbv = g.nb;
      // the previous group's MMAs have all completed: this thread consumed their last
      // accumulator; the issuer waits for all epilogue threads before the next group
      write_query_planes<G>(QI, q, qt, nqv, gg, g.hq, tid);
      fence_proxy_async_smem();
      mbar_arrive(&bars->q_full);
      if (tid < kN) {
        Ts[tid] = tid < nqv ? tinit[(qt * kN + tid) * g.hkv + gg] : CUDART_INF_F;
        cnt[tid] = 0;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
      // this CTA's segments of group gg: [hkv][CTA slot][query][kSegCap]
      const int64_t slot = (int64_t)blockIdx.x - ((int64_t)gg * g.nch) / g.per;
      const int64_t seg0 = ((int64_t)gg * g.ns_max + slot) * g.nq_pad + qt * kN;
      for (; u < ue; ++u, ++tile) {
        const int a = (int)(tile % NACC);
        if (!aborted && __any_sync(0xffffffffu, *abort_flag != 0)) aborted = true;
        if (!aborted && !mbar_wait_warp(&bars->acc_full[a], (uint32_t)(tile / NACC) & 1)) {
          fail();
          aborted = true;
        }
        if (aborted) continue;
        tc_fence_after();
        uint32_t v[32];
        load_scores<HI>(lane_base + a * ACOLS, v);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->acc_empty[a]);   // the scores are in registers
        const int64_t j = (u % g.nch) * g.stride * kM + quarter * 32 + lane;
        uint32_t pm = pass_mask(v, Ts + qh * 32);
        if (j >= nbv || nq_here <= 0) pm = 0u;
        else if (nq_here < 32) pm &= (1u << nq_here) - 1u;
        // each lane appends its own passes (a block passes for few queries, so the
        // lanes' loops are short), one shared-memory slot reservation per key
        while (pm != 0u) {
          const int n = __ffs(pm) - 1;
          pm &= pm - 1u;
          const int pos = atomicAdd(&cnt[qh * 32 + n], 1);
          if (pos < kSegCap)
            cand[(seg0 + qh * 32 + n) * kSegCap + pos] = make_key(__uint_as_float(pick32(v, n)), j);
        }
      }
      // the group's keys are all in: publish the counts (beyond kSegCap: overflowed)
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
      if (tid < kN) g.seg_count[seg0 + tid] = aborted ? 0 : cnt[tid];
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 0-7)
    uint64_t y[kOwned];                           // lists of queries warp + 8 i
    float T[kOwned];
    int c[kOwned];
#pragma unroll
    for (int i = 0; i < kOwned; ++i) { y[i] = 0ull; T[i] = -CUDART_INF_F; c[i] = 0; }
    const int quarter = warp & 3, qh = warp >> 2;   // TMEM lanes 32*quarter.., queries 32*qh..
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16) + qh * 32;
    const uint32_t lt_mask = (1u << lane) - 1u;
    bool aborted = false;
    int64_t tile = 0;
    int64_t u = u0;
    while (u < u1) {
      const int gg = (int)(u / g.nch);
      const int64_t ue = ((int64_t)gg + 1) * g.nch < u1 ? ((int64_t)gg + 1) * g.nch : u1;
      const int64_t nbv = g.nb;                                             // valid blocks
      // group-summed query planes of group gg (the previous group's MMAs have all
      // completed: this thread consumed their last accumulator)
      write_query_planes<G>(QI, q, qt, nqv, gg, g.hq, tid);
      fence_proxy_async_smem();
      mbar_arrive(&bars->q_full);
      if (tinit != nullptr) {
        // a valid starting bound: 32 sampled blocks of this group score at least T0
#pragma unroll
        for (int i = 0; i < kOwned; ++i) {
          const int n = warp + kEpiWarps * i;
          T[i] = n < nqv ? tinit[(qt * kN + n) * g.hkv + gg] : -CUDART_INF_F;
          if (lane == 0) Ts[n] = T[i];
        }
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");

      for (; u < ue; ++u, ++tile) {
        const int a = (int)(tile % NACC);
        if (!aborted && __any_sync(0xffffffffu, *abort_flag != 0)) aborted = true;
        if (!aborted && !mbar_wait_warp(&bars->acc_full[a], (uint32_t)(tile / NACC) & 1)) {
          fail();
          aborted = true;
        }
        if constexpr (GMAX) {
          if (!aborted) {
            tc_fence_after();
            uint32_t v[32];
            load_scores<HI>(lane_base + a * ACOLS, v);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->acc_empty[a]);
            const int64_t j = (u % g.nch) * g.stride * kM + quarter * 32 + lane;
            const bool valid = j < nbv;
            uint32_t mine = 0u;                   // lane n: group max of query 32*qh + n
#pragma unroll
            for (int n = 0; n < 32; ++n) {
              const uint32_t m =
                  __reduce_max_sync(0xffffffffu, valid ? score_ord(__uint_as_float(v[n])) : 0u);
              if (lane == n) mine = m;
            }
            const int qn = qh * 32 + lane;
            if (qn < nqv)
              gmax[((qt * kN + qn) * g.hkv + gg) * (g.nch * 4) + (u % g.nch) * 4 + quarter] = mine;
          }
          continue;
        }
        if (!aborted) {
          tc_fence_after();
          uint32_t v[32];
          tmem_ld32(lane_base + a * ACOLS, v);
          tmem_ld_wait();
          const int64_t j = (u % g.nch) * g.stride * kM + quarter * 32 + lane;
          const bool valid = j < nbv;
          // bit n: this block reaches T of query 32*qh + n
          uint32_t pm = pass_mask(v, Ts + qh * 32);
          const int nq_here = nqv - qh * 32;       // valid queries of this warp's 32
          if (!valid || nq_here <= 0) pm = 0u;
          else if (nq_here < 32) pm &= (1u << nq_here) - 1u;
          if (__any_sync(0xffffffffu, pm != 0u)) {
            // lane n takes query 32*qh + n: transpose the 32x32 pass matrix (lanes =
            // blocks, bits = queries), reserve that query's slots with one atomic per
            // lane, then every block stores its keys at base + rank among the passes
            const uint32_t mt = transpose32(pm, lane);
            const int nmine = __popc(mt);
            int base = 0;
            if (nmine > 0) base = atomicAdd(&cnt[qh * 32 + lane], nmine);
            uint32_t any = __ballot_sync(0xffffffffu, nmine > 0);   // queries with passes
            while (any != 0u) {
              // the score column of query n is re-read from TMEM (a uniform column index)
              const int n = __ffs(any) - 1;
              any &= any - 1u;
              const bool pass = (pm >> n) & 1u;
              const uint32_t mn = __ballot_sync(0xffffffffu, pass);
              const int bn = __shfl_sync(0xffffffffu, base, n);
              const uint32_t sv = tmem_ld1(lane_base + a * ACOLS + n);
              tmem_ld_wait();
              if (pass)
                pend[(size_t)(qh * 32 + n) * kPend + bn + __popc(mn & lt_mask)] =
                    make_key(__uint_as_float(sv), j);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->acc_empty[a]);
        }
        // every warp's appends of this chunk are in; owners merge, then republish T
        asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
        if (!aborted) {
          int need = 0;
#pragma unroll
          for (int i = 0; i < kOwned; ++i) {
            c[i] = cnt[warp + kEpiWarps * i];
            need |= c[i] >= 32;
          }
          if (need) {
            do {
              joint_drain(y, T, c, pend, warp, lane);
              need = 0;
#pragma unroll
              for (int i = 0; i < kOwned; ++i) need |= c[i] >= 32;
            } while (need);
            if (lane == 0) {
#pragma unroll
              for (int i = 0; i < kOwned; ++i) {
                cnt[warp + kEpiWarps * i] = c[i];
                Ts[warp + kEpiWarps * i] = T[i];
              }
            }
          }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
      }
      if constexpr (GMAX) continue;
      // end of this group's range: flush the lists to this CTA's slot of group gg
      if (!aborted) {
        int any = 0;
#pragma unroll
        for (int i = 0; i < kOwned; ++i) {
          c[i] = cnt[warp + kEpiWarps * i];
          any |= c[i];
        }
        if (any) joint_drain(y, T, c, pend, warp, lane);
      }
      const int64_t c_first = ((int64_t)gg * g.nch) / g.per;
      const int64_t slot = (int64_t)blockIdx.x - c_first;
#pragma unroll
      for (int i = 0; i < kOwned; ++i) {
        const int n = warp + kEpiWarps * i;
        if (n < nqv) {
          const int64_t row = ((int64_t)gg * g.ns_max + slot) * g.nq_pad + qt * kN + n;
          cand[row * kList + lane] = aborted ? 0ull : y[i];
        }
        if (lane == 0) { cnt[n] = 0; Ts[n] = -CUDART_INF_F; }
        y[i] = 0ull;
        T[i] = -CUDART_INF_F;
        c[i] = 0;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kAcc * kN);
  }
}

// A row's best topk from its keys y (sorted descending over lanes, 0 = empty): the block
// indices ascending (-1 padded) into idx, or, when `keys` is given, the keys themselves
// with their block index moved up by `block_offset` (empty entries stay 0).
__device__ __forceinline__ void write_selection(uint64_t y, int lane, int64_t w, int topk,
                                                int32_t* __restrict__ idx,
                                                uint64_t* __restrict__ keys,
                                                int64_t block_offset) {
  const int blk = y != 0ull ? key_block(y) : -1;
  if (keys != nullptr) {
    if (lane < topk) {
      const uint32_t jg = (uint32_t)((int64_t)blk + block_offset);
      keys[w * topk + lane] = y == 0ull ? 0ull : ((y & 0xffffffff00000000ull) | (uint32_t)~jg);
    }
    return;
  }
  // ascending by block index (empty entries sort last)
  int j = (lane < topk && blk >= 0) ? blk : 0x7fffffff;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      const int p = __shfl_xor_sync(0xffffffffu, j, jj);
      const bool take_min = ((lane & jj) == 0) == ((lane & k) == 0);
      j = take_min ? min(j, p) : max(j, p);
    }
  }
  if (lane < topk) idx[w * topk + lane] = j == 0x7fffffff ? -1 : j;
}

// Two warps per block, one per (query, group) row of a filtered scan: the row's best kq
// of its n candidates, gathered from the row's segments (one per CTA that scanned the
// group).  The keys sit in registers (kFilterCap / 32 per lane); the kq-th
// largest is found bit by bit, first on the score bits, then (only when scores tie at
// the cut) on the block bits; the keys at or above it are the selection (distinct).
// CANDS = false: kq = topk, written as the list merge writes it; CANDS = true: kq =
// kCand, the candidates' blocks (any order) and amin = the score of the kq-th.
// A row with an overflowed segment, more than kFilterCap candidates or fewer than kq is
// not selected here: *fail = 1 and the exact list scan redoes every row.
template <bool CANDS>
__global__ void __launch_bounds__(64)
filter_select_kernel(const uint64_t* __restrict__ fc, DecGeom g, int32_t* __restrict__ idx,
                     uint64_t* __restrict__ keys, int64_t block_offset,
                     int32_t* __restrict__ acand, float* __restrict__ amin, int* fail) {
  constexpr int R = kFilterCap / 32;
  __shared__ int soff[2][kMaxSegments];
  __shared__ uint64_t sel[2][kCand];
  const int wib = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t w = (int64_t)blockIdx.x * 2 + wib;
  if (w >= g.n_query * g.hkv) return;
  const int topk = g.topk;
  const int kq = CANDS ? kCand : topk;
  const int64_t nq = w / g.hkv;
  const int gg = (int)(w % g.hkv);
  // the row's segments: one per CTA that scanned part of group gg
  const int64_t c_first = ((int64_t)gg * g.nch) / g.per;
  int64_t c_last = (((int64_t)gg + 1) * g.nch - 1) / g.per;
  if (c_last > g.ncta_x - 1) c_last = g.ncta_x - 1;
  // segment offsets: lane c reads the count of segment c (32 at a time), an inclusive
  // scan places them; so[s] = first key of segment s in the row's list
  int* so = soff[wib];
  const int nseg = (int)(c_last - c_first + 1);
  int n = 0;
  bool over = false;
  for (int c0 = 0; c0 < nseg; c0 += 32) {
    const int c = c0 + lane;
    const int m = c < nseg ? g.seg_count[((int64_t)gg * g.ns_max + c) * g.nq_pad + nq] : 0;
    over |= __any_sync(0xffffffffu, m > kSegCap);
    int inc = m;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += t;
    }
    if (c < nseg) so[c] = n + inc - m;
    n += __shfl_sync(0xffffffffu, inc, 31);
  }
  if (over || n > kFilterCap || n < kq) {
    if (lane == 0) *fail = 1;
    return;
  }
  __syncwarp();
  const int nr = (n + 31) / 32;                   // registers in use (warp-uniform)
  // key p of the row's list: a binary search for its segment, then one load (all loads
  // independent, so they overlap)
  uint64_t kk[R];
#pragma unroll
  for (int i = 0; i < R; ++i) {
    kk[i] = 0ull;
    const int p = lane + 32 * i;
    if (i < nr && p < n) {
      int lo = 0, hi = nseg - 1;                    // last segment with so[s] <= p
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (so[mid] <= p) lo = mid; else hi = mid - 1;
      }
      const int64_t seg = ((int64_t)gg * g.ns_max + lo) * g.nq_pad + nq;
      kk[i] = __ldg(fc + seg * kSegCap + (p - so[lo]));
    }
  }
  // the kq-th largest score bits P
  uint32_t P = 0u;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t c = P | (1u << bit);
    int cnt = 0;
#pragma unroll
    for (int i = 0; i < R; ++i)
      if (i < nr) cnt += (uint32_t)(kk[i] >> 32) >= c;
    if (__reduce_add_sync(0xffffffffu, cnt) >= (unsigned)kq) P = c;
  }
  int ge = 0, gt = 0;
#pragma unroll
  for (int i = 0; i < R; ++i) {
    if (i < nr) {
      ge += (uint32_t)(kk[i] >> 32) >= P;
      gt += (uint32_t)(kk[i] >> 32) > P;
    }
  }
  ge = (int)__reduce_add_sync(0xffffffffu, ge);
  gt = (int)__reduce_add_sync(0xffffffffu, gt);
  uint64_t thr = (uint64_t)P << 32;
  if (ge > kq) {                                  // scores tie at the cut: the block bits
    const int need = kq - gt;
    uint32_t Lb = 0u;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t c = Lb | (1u << bit);
      int cnt = 0;
#pragma unroll
      for (int i = 0; i < R; ++i)
        if (i < nr) cnt += (uint32_t)(kk[i] >> 32) == P && (uint32_t)kk[i] >= c;
      if (__reduce_add_sync(0xffffffffu, cnt) >= (unsigned)need) Lb = c;
    }
    thr |= Lb;
  }
  // gather the kq keys >= thr (warp-ordered by an exclusive scan of per-lane counts)
  int m = 0;
#pragma unroll
  for (int i = 0; i < R; ++i)
    if (i < nr) m += kk[i] >= thr;
  int off = m;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, off, o);
    if (lane >= o) off += t;
  }
  off -= m;
#pragma unroll
  for (int i = 0; i < R; ++i)
    if (i < nr && kk[i] >= thr) sel[wib][off++] = kk[i];
  __syncwarp();
  if (CANDS) {
    for (int p = lane; p < kCand; p += 32) acand[w * kCand + p] = key_block(sel[wib][p]);
    if (lane == 0) amin[w] = key_score(thr);
    return;
  }
  uint64_t y = lane < kq ? sel[wib][lane] : 0ull;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {             // bitonic sort, descending
#pragma unroll
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      const uint64_t p = __shfl_xor_sync(0xffffffffu, y, jj);
      const bool take_max = ((lane & jj) == 0) == ((lane & k) == 0);
      y = take_max ? umax64(y, p) : umin64(y, p);
    }
  }
  write_selection(y, lane, w, topk, idx, keys, block_offset);
}

// eps of a row's certificate: (max ||lo_j|| + 2^-9 max ||hi_j||) ||Q|| with 1% slack, Q
// the group-summed query (fp32, the sum the scan splits); warp-collective.
__device__ __forceinline__ float row_eps(const __nv_bfloat16* __restrict__ q,
                                         const float* __restrict__ bounds, int64_t n, int gg,
                                         int hq, int G, int hkv, int lane) {
  const __nv_bfloat16* qr = q + (n * hq + (int64_t)gg * G) * kD + lane * 4;
  float a[4] = {0.f, 0.f, 0.f, 0.f};
  for (int h = 0; h < G; ++h) {
    const uint2 raw = *reinterpret_cast<const uint2*>(qr + (int64_t)h * kD);
    a[0] += bf16lo_to_f32(raw.x);
    a[1] += bf16hi_to_f32(raw.x);
    a[2] += bf16lo_to_f32(raw.y);
    a[3] += bf16hi_to_f32(raw.y);
  }
  float sq = a[0] * a[0] + a[1] * a[1] + a[2] * a[2] + a[3] * a[3];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  return (bounds[gg] + 0x1p-9f * bounds[hkv + gg]) * sqrtf(sq) * 1.01f;
}

// Exact rescoring of the candidates, two rows (queries 2p, 2p + 1 of query tile qt,
// group gg) per CTA: the rows' 2 x kCand candidate blocks are gathered from the encoded
// planes into one 128-row A tile (hi and lo), scored against the tile's query planes with
// the scan's three-term MMAs (M = 128, N = 64, the same k-step order), and each row reads
// its query's column: the exact scores of its candidates, bitwise the full scan's.  The
// row's best topk then gets its certificate (see launch_topk_decode_tc) and is written.
constexpr int kRsThreads = 256;
struct __align__(8) RBars {
  uint64_t mma_done;
  uint32_t tmem_base;
};
constexpr size_t rescore_smem() { return 1024 + 4 * (size_t)kPlane + kQBytes + sizeof(RBars); }

template <int G>
__global__ void __launch_bounds__(kRsThreads)
rescore_kernel(const unsigned char* __restrict__ ktiles, int64_t nch_full,
               const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ acand,
               const float* __restrict__ amin, const float* __restrict__ bounds,
               int32_t* __restrict__ idx, uint64_t* __restrict__ keys, int64_t block_offset,
               int* fail, int* err, DecGeom g) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* AH = base;                           // [half][128 rows][128 B], hi
  unsigned char* AL = AH + 2 * kPlane;                // lo
  unsigned char* QI = AL + 2 * kPlane;                // query planes of the tile
  RBars* bars = reinterpret_cast<RBars*>(QI + kQBytes);
  __shared__ uint64_t rk[2][kCand];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int gg = blockIdx.y;
  const int64_t qt = blockIdx.z;
  const int nqv = (int)(g.n_query - qt * kN < kN ? g.n_query - qt * kN : kN);
  const int n0 = 2 * blockIdx.x;
  if (n0 >= nqv) return;                              // uniform for the CTA
  if (tid == 0) {
    mbar_init(&bars->mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 0) { tmem_alloc(&bars->tmem_base, kN); tmem_relinquish(); }
  write_query_planes<G, kRsThreads>(QI, q, qt, nqv, gg, g.hq, tid);
  // gather: 128 rows x (2 planes x 2 halves x 8 chunks of 16 B), 8 loads in flight each
  const size_t plane = (size_t)g.hkv * nch_full * 2 * kPlane;
  static_assert((128 * 32) % (kRsThreads * 8) == 0, "gather split");
#pragma unroll 1
  for (int e0 = tid; e0 < 128 * 32; e0 += kRsThreads * 8) {
    uint4 val[8];
    int64_t dst[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int e = e0 + k * kRsThreads;
      const int r = e >> 5, lc = e & 7, hf = (e >> 3) & 1, pl = (e >> 4) & 1;
      const int n = n0 + (r >> 6);
      const int64_t row = (qt * kN + n) * g.hkv + gg;
      const int j = n < nqv ? acand[row * kCand + (r & 63)] : -1;
      val[k] = make_uint4(0u, 0u, 0u, 0u);
      if (j >= 0 && j < g.nb) {
        const size_t src = (size_t)pl * plane +
                           (((size_t)gg * nch_full + j / kM) * 2 + hf) * kPlane +
                           (size_t)(j % kM) * 128 + (size_t)((lc ^ (j & 7)) << 4);
        val[k] = ldg16(ktiles + src);
      }
      dst[k] = (int64_t)pl * 2 * kPlane + hf * kPlane + r * 128 + ((lc ^ (r & 7)) << 4);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) *reinterpret_cast<uint4*>(AH + dst[k]) = val[k];
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  if (tid == 0) {
    constexpr uint32_t idesc = idesc_bf16(kM, kN, 0, 0);
    const uint64_t qd = sdesc_sw128(smem_u32(QI), 16, 1024);
    const uint64_t ad = sdesc_sw128(smem_u32(AH), 16, 1024);
    for (int hf = 0; hf < 2; ++hf) {
      const uint64_t kh = ad + (uint64_t)((hf * kPlane) >> 4);
      const uint64_t kl = kh + (uint64_t)((2 * kPlane) >> 4);
      const uint64_t qh = qd + (uint64_t)((2 * hf * kQHalf) >> 4);
      const uint64_t ql = qd + (uint64_t)(((2 * hf + 1) * kQHalf) >> 4);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t o = (uint64_t)(ks * 2);
        umma_ss(tmem, kh + o, qh + o, idesc, (hf | ks) ? 1u : 0u);
        umma_ss(tmem, kh + o, ql + o, idesc, 1u);
        umma_ss(tmem, kl + o, qh + o, idesc, 1u);
      }
    }
    umma_commit(&bars->mma_done);
  }
  // warps 0-3 hold TMEM lanes 32w..: candidates 32(w%2).. of row n0 + w/2
  const int rsel = (warp & 3) >> 1;
  const int n = n0 + rsel;
  if (warp < 4) {
    const bool ok = mbar_wait_warp(&bars->mma_done, 0);
    if (!ok && lane == 0) set_device_error(err, MSA_DEVERR_TIMEOUT);
    tc_fence_after();
    uint32_t sv = 0u;
    if (ok) sv = tmem_ld1(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(n < nqv ? n : n0));
    tmem_ld_wait();
    const int c = (warp & 1) * 32 + lane;
    const int64_t row = (qt * kN + n) * g.hkv + gg;
    const int j = (ok && n < nqv) ? acand[row * kCand + c] : -1;
    rk[rsel][c] = (j >= 0 && j < g.nb) ? make_key(__uint_as_float(sv), j) : 0ull;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kN);
  }
  if (warp >= 4 || (warp & 1) != 0 || n >= nqv) return;   // warps 0 and 2: one row each
  uint64_t z0 = rk[rsel][lane], z1 = rk[rsel][32 + lane];
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {                 // both halves sorted descending
#pragma unroll
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      const uint64_t p0 = __shfl_xor_sync(0xffffffffu, z0, jj);
      const uint64_t p1 = __shfl_xor_sync(0xffffffffu, z1, jj);
      const bool take_max = ((lane & jj) == 0) == ((lane & k) == 0);
      z0 = take_max ? umax64(z0, p0) : umin64(z0, p0);
      z1 = take_max ? umax64(z1, p1) : umin64(z1, p1);
    }
  }
  z1 = __shfl_sync(0xffffffffu, z1, 31 - lane);       // z0 ++ reversed z1 is bitonic
  warp_sort_bitonic64(z0, z1, lane);
  const int64_t row = (qt * kN + n) * g.hkv + gg;
  // certificate: every block outside the candidates scores at most amin + eps
  const float sk = key_score(__shfl_sync(0xffffffffu, z0, g.topk - 1));
  const float am = amin[row];
  const float eps = row_eps(q, bounds, qt * kN + n, gg, g.hq, G, g.hkv, lane);
  if (!(am == -CUDART_INF_F || sk > am + eps) && lane == 0) *fail = 1;
  write_selection(z0, lane, row, g.topk, idx, keys, block_offset);
}

// One warp per (query, group): merges the sorted lists of the CTAs that covered the
// group, then writes the best `topk` block indices ascending (-1 padded) or, when `keys`
// is given, the best `topk` keys sorted descending with their block index moved up by
// `block_offset` (a shard's blocks renumbered to bank-wide ids; empty entries stay 0).
__global__ void topk_decode_merge_kernel(const uint64_t* __restrict__ cand,
                                         int32_t* __restrict__ idx, uint64_t* __restrict__ keys,
                                         int64_t block_offset, DecGeom g) {
  if (g.run_if != nullptr && *(volatile const int*)g.run_if == 0) return;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (w >= g.n_query * g.hkv) return;
  const int64_t n = w / g.hkv;
  const int gg = (int)(w % g.hkv);
  const int64_t c_first = ((int64_t)gg * g.nch) / g.per;
  int64_t c_last = (((int64_t)gg + 1) * g.nch - 1) / g.per;
  if (c_last > g.ncta_x - 1) c_last = g.ncta_x - 1;
  uint64_t y = 0ull;
  const uint64_t* src = cand + ((int64_t)gg * g.ns_max * g.nq_pad + n) * kList + lane;
  const int64_t step = g.nq_pad * kList;            // next CTA slot of the group
  const int nl = (int)(c_last - c_first + 1);
  // the next list loads while the current one merges
  uint64_t x = nl > 0 ? __ldg(src) : 0ull;
  for (int c = 0; c < nl; ++c) {
    const uint64_t xn = c + 1 < nl ? __ldg(src + (c + 1) * step) : 0ull;
    y = warp_merge_desc(y, x, lane);
    x = xn;
  }
  write_selection(y, lane, w, g.topk, idx, keys, block_offset);
}

// One warp per (query, group): T0 = the rank-th largest of the sampled 32-block group
// maxima (a valid bound: `rank` different blocks score at least T0), found bit by bit on
// the order-preserving bits; -inf when fewer than `rank` groups were sampled.
constexpr int kThrRegs = 24;                    // register path up to 768 group maxima

// It also clears the failure flag for the passes that follow.
__global__ void sample_threshold_kernel(const uint32_t* __restrict__ gmax, float* __restrict__ tout,
                                        int64_t rows, int ngroups, uint32_t rank, int* fail) {
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (blockIdx.x == 0 && threadIdx.x == 0) *fail = 0;
  if (w >= rows) return;
  const uint32_t* vals = gmax + w * ngroups;
  uint32_t prefix = 0u;
  if (ngroups <= 32 * kThrRegs) {
    uint32_t r[kThrRegs];                       // this lane's values, loaded once
#pragma unroll
    for (int k = 0; k < kThrRegs; ++k) {
      const int i = lane + 32 * k;
      r[k] = i < ngroups ? __ldg(vals + i) : 0u;
    }
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = prefix | (1u << bit);
      uint32_t c = 0;
#pragma unroll
      for (int k = 0; k < kThrRegs; ++k) c += r[k] >= cand;
      if (__reduce_add_sync(0xffffffffu, c) >= rank) prefix = cand;
    }
  } else {
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = prefix | (1u << bit);
      uint32_t c = 0;
      for (int i = lane; i < ngroups; i += 32) c += __ldg(vals + i) >= cand;
      if (__reduce_add_sync(0xffffffffu, c) >= rank) prefix = cand;
    }
  }
  if (lane == 0) tout[w] = ord_score(prefix);
}

// Sample pass: every kSampleStride-th chunk, when the bank has at least kSampleMinChunks
// chunks per group (the sample then holds >= 16 chunks, 64 block groups, per group: enough
// for a bound on the 32nd and on the kCand-th best).
constexpr int64_t kSampleStride = 8;
constexpr int64_t kSampleMinChunks = 128;

DecGeom make_dgeom(const Shape& s, int64_t n_query, int64_t stride) {
  DecGeom g{};
  g.nb = s.nb;
  g.n_query = n_query;
  g.stride = stride;
  g.nch_full = (s.nb + kM - 1) / kM;
  g.nch = (g.nch_full + stride - 1) / stride;
  const int64_t qtiles = (n_query + kN - 1) / kN;
  g.nq_pad = qtiles * kN;
  const int sms = sm_count();
  int64_t ncx = sms / qtiles;
  if (ncx < 1) ncx = 1;
  const int64_t total = s.hkv * g.nch;
  if (ncx > total) ncx = total;
  g.per = (total + ncx - 1) / ncx;
  g.ncta_x = (int)((total + g.per - 1) / g.per);
  int64_t ns = (g.nch + g.per - 1) / g.per + 1;
  if (ns > g.ncta_x) ns = g.ncta_x;
  g.ns_max = (int)ns;
  g.hq = (int)s.hq;
  g.hkv = (int)s.hkv;
  g.G = (int)(s.hq / s.hkv);
  g.topk = (int)s.topk;
  return g;
}

bool use_sample(const Shape& s) { return (s.nb + kM - 1) / kM >= kSampleMinChunks; }

template <int G, int MODE>
cudaError_t run_scan_g(const DecGeom& g, const CUtensorMap& mh, const CUtensorMap& ml,
                       const void* kt, const void* q, const float* tinit, uint64_t* cand,
                       uint32_t* gmax, int* err, cudaStream_t st) {
  const size_t smem = smem_bytes(MODE);
  cudaError_t e = cudaFuncSetAttribute(topk_decode_tc_kernel<G, MODE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)g.ncta_x, (unsigned)(g.nq_pad / kN));
  topk_decode_tc_kernel<G, MODE><<<grid, kThreads, smem, st>>>(
      mh, ml, (const unsigned char*)kt, (const __nv_bfloat16*)q, tinit, cand, gmax, err, g);
  return cudaGetLastError();
}

template <int MODE>
cudaError_t run_scan(const DecGeom& g, const CUtensorMap& mh, const CUtensorMap& ml,
                     const void* kt, const void* q, const float* tinit, uint64_t* cand,
                     uint32_t* gmax, int* err, cudaStream_t st) {
  switch (g.G) {
    case 1: return run_scan_g<1, MODE>(g, mh, ml, kt, q, tinit, cand, gmax, err, st);
    case 2: return run_scan_g<2, MODE>(g, mh, ml, kt, q, tinit, cand, gmax, err, st);
    case 4: return run_scan_g<4, MODE>(g, mh, ml, kt, q, tinit, cand, gmax, err, st);
    default: return run_scan_g<8, MODE>(g, mh, ml, kt, q, tinit, cand, gmax, err, st);
  }
}

// Candidate lists [hkv][CTA slot][query][list] of one scan geometry.
size_t cand_bytes(const DecGeom& g, int list) {
  return (size_t)g.hkv * g.ns_max * g.nq_pad * list * sizeof(uint64_t);
}

// Workspace: one list region (the largest of the passes' candidate lists or filter
// segments), the sample thresholds [query][hkv], the segment counts, the
// sampled group maxima [query][hkv][group], and for the certified selection of an
// encoded bank: the row candidates [query][hkv][kCand], their last hi-plane scores
// [query][hkv] and the failure flag.
struct DecWs {
  size_t cand, tinit, segc, gmax, acand, amin, small, total;
};
size_t up256(size_t x) { return (x + 255) / 256 * 256; }
DecWs dec_ws(const Shape& s, int64_t n_query) {
  const DecGeom g = make_dgeom(s, n_query, 1);
  size_t lists = cand_bytes(g, kList);
  const size_t lf = cand_bytes(g, kSegCap);                 // filter segments
  if (use_sample(s) && lf > lists) lists = lf;
  DecWs w{};
  size_t o = 0;
  w.cand = o;   o += up256(lists);
  w.tinit = o;  o += up256((size_t)n_query * s.hkv * sizeof(float));
  w.segc = o;   o += up256(cand_bytes(g, 1) / sizeof(uint64_t) * sizeof(int));
  w.gmax = o;
  if (use_sample(s)) {
    const DecGeom gs = make_dgeom(s, n_query, kSampleStride);
    o += up256((size_t)n_query * s.hkv * gs.nch * 4 * sizeof(uint32_t));
  }
  w.acand = o;  o += up256((size_t)n_query * s.hkv * kCand * 4);
  w.amin = o;   o += up256((size_t)n_query * s.hkv * 4);
  w.small = o;  o += 256;                                                 // failure flag
  w.total = o;
  return w;
}

template <int G>
cudaError_t run_rescore_g(const Shape& s, const DecGeom& g, const void* kt, const void* q,
                          const int32_t* acand, const float* amin, const float* bounds,
                          int32_t* idx, uint64_t* keys, int64_t block_offset, int* fail,
                          int* err, cudaStream_t st) {
  const size_t smem = rescore_smem();
  cudaError_t e = cudaFuncSetAttribute(rescore_kernel<G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)(kN / 2), (unsigned)s.hkv, (unsigned)(g.nq_pad / kN));
  rescore_kernel<G><<<grid, kRsThreads, smem, st>>>(
      (const unsigned char*)kt, g.nch_full, (const __nv_bfloat16*)q, acand, amin, bounds, idx,
      keys, block_offset, fail, err, g);
  return cudaGetLastError();
}

}  // namespace

bool tc_decode_supported(const Shape& s) {
  if (s.dtype != MSA_BF16 || s.d != kD) return false;
  const int64_t G = s.hq / s.hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return false;
  if (s.topk > kList) return false;
  if (s.nb >= ((int64_t)1 << 31) - kM) return false;        // TMA row coordinate, key
  if (s.hkv * kD > ((int64_t)1 << 31)) return false;
  if (s.hkv > kMaxBoundGroups) return false;                 // bounds of the encoded planes
  return true;
}

size_t topk_decode_tc_ws_bytes(const Shape& s, int64_t n_query) {
  return dec_ws(s, n_query).total;
}

// Selection of a bank given as tensor-map planes (natural layout) or as an encoded image
// (kbar_tiles), exact under (score desc, block asc) with the score of the three-term
// split product.
//
// Banks of at least kSampleMinChunks chunks per group first run the sample pass: its
// bound per row has at least `rank` blocks at or above it.  When the bound is tight (it
// ranks within the top eighth of the sampled group maxima), the full scan runs as a
// filter (every score >= the bound into the row's segments, no lists, no barriers
// between the epilogue warps) followed by a per-row selection; a row whose segments
// overflow falls back to the list scan.  Otherwise the list scan runs, started from the
// bound when there is one.
//
// An encoded image that allows the filter at rank kCand gets a certified selection that
// reads the lo plane only for candidates:
//   1. the hi-plane filter: each row's best kCand blocks by the two-term score
//      a_j = Khi_j . (Qhi + Qlo), and amin = a of the last one;
//   2. the exact (three-term) scores of each row's candidates, from the same MMAs as the
//      full scan, and the certificate: the exact score differs from a_j by Klo_j . Qhi
//      plus the two accumulations' rounding, so |exact_j - a_j| <= eps = (max ||lo_j|| +
//      2^-9 max ||hi_j||) ||Q|| (with 1% slack; both maxima are stored with the image).
//      Every block outside the row's candidates then scores at most amin + eps; when the
//      candidates' k-th best exact score lies strictly above that, no other block can
//      enter the top k, and the candidates' top k is the bank's;
//   3. if any row failed (near-equal scores over a wide range, e.g. exact ties, or a
//      filter overflow), the three-term list scan of the whole bank and its merge run as
//      well and overwrite every row; otherwise both launches exit at once.
// Exact scores come from the same three-term MMAs in the rescoring, the filter and the
// list scans, so the selection is the natural-layout one.
cudaError_t launch_topk_decode_tc(const Shape& s, int64_t n_query, const void* q,
                                  const void* kbar_hi, const void* kbar_lo,
                                  const void* kbar_tiles, int32_t* idx, void* ws, int* err,
                                  cudaStream_t st, uint64_t* keys, int64_t block_offset) {
  CUtensorMap mh{}, ml{};
  if (kbar_tiles == nullptr && (!make_bf16_2d_map(&mh, kbar_hi, s.nb, s.hkv * kD, kM) ||
                                !make_bf16_2d_map(&ml, kbar_lo, s.nb, s.hkv * kD, kM)))
    return cudaErrorInvalidValue;
  const void* kt = kbar_tiles;
  DecGeom g = make_dgeom(s, n_query, 1);
  const DecWs L = dec_ws(s, n_query);
  char* base = reinterpret_cast<char*>(ws);
  uint64_t* cand = reinterpret_cast<uint64_t*>(base + L.cand);
  float* tinit = reinterpret_cast<float*>(base + L.tinit);
  int* segc = reinterpret_cast<int*>(base + L.segc);
  uint32_t* gmax = reinterpret_cast<uint32_t*>(base + L.gmax);
  int* fail = reinterpret_cast<int*>(base + L.small);
  const int64_t rows = n_query * s.hkv;
  const unsigned merge_blocks = (unsigned)((rows + 1) / 2);   // two warps per block
  // the filter needs a tight start: the sample's bound must rank among the top eighth of
  // its group maxima (else a row's candidates would approach kFilterCap), and the
  // selection's segment offsets must fit
  const bool sample = use_sample(s);
  const DecGeom gs = make_dgeom(s, n_query, kSampleStride);
  const int64_t maxima = sample ? gs.nch * 4 : 0;
  const bool fits = sample && g.ns_max <= kMaxSegments;
  const bool certified = kbar_tiles != nullptr && fits && maxima >= 8 * kCand;
  const bool filter = certified || (fits && maxima >= 8 * kList);
  cudaError_t e;
  if (sample) {
    // every 8th chunk first: the 32nd (kCand-th) largest of its 32-block group maxima
    // per (query, group) is a valid bound that starts the full scan
    e = certified ? run_scan<kModeSample | kModeHi>(gs, mh, ml, kt, q, nullptr, nullptr, gmax,
                                                    err, st)
                  : run_scan<kModeSample>(gs, mh, ml, kt, q, nullptr, nullptr, gmax, err, st);
    if (e != cudaSuccess) return e;
    sample_threshold_kernel<<<merge_blocks, 64, 0, st>>>(gmax, tinit, rows, (int)(gs.nch * 4),
                                                         certified ? kCand : kList, fail);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const float* t0 = sample ? tinit : nullptr;
  DecGeom gf = g;
  gf.seg_count = segc;
  if (!certified) {
    if (!filter) {
      if ((e = run_scan<0>(g, mh, ml, kt, q, t0, cand, nullptr, err, st)) != cudaSuccess)
        return e;
      topk_decode_merge_kernel<<<merge_blocks, 64, 0, st>>>(cand, idx, keys, block_offset, g);
      return cudaGetLastError();
    }
    if ((e = run_scan<kModeFilter>(gf, mh, ml, kt, q, t0, cand, nullptr, err, st)) !=
        cudaSuccess)
      return e;
    filter_select_kernel<false><<<merge_blocks, 64, 0, st>>>(cand, gf, idx, keys, block_offset,
                                                             nullptr, nullptr, fail);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    g.run_if = fail;                                  // overflow: the list scan
    if ((e = run_scan<0>(g, mh, ml, kt, q, t0, cand, nullptr, err, st)) != cudaSuccess) return e;
    topk_decode_merge_kernel<<<merge_blocks, 64, 0, st>>>(cand, idx, keys, block_offset, g);
    return cudaGetLastError();
  }
  // 1. hi-plane candidates
  int32_t* acand = reinterpret_cast<int32_t*>(base + L.acand);
  float* amin = reinterpret_cast<float*>(base + L.amin);
  if ((e = run_scan<kModeFilter | kModeHi>(gf, mh, ml, kt, q, t0, cand, nullptr, err, st)) !=
      cudaSuccess)
    return e;
  filter_select_kernel<true><<<merge_blocks, 64, 0, st>>>(cand, gf, nullptr, nullptr, 0, acand,
                                                          amin, fail);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // 2. the candidates' exact scores, each row's certificate and selection
  const float* bounds = reinterpret_cast<const float*>(
      reinterpret_cast<const char*>(kbar_tiles) + bank_kbar_planes_bytes(s) * 2);
  switch (g.G) {
    case 1: e = run_rescore_g<1>(s, g, kt, q, acand, amin, bounds, idx, keys, block_offset,
                                  fail, err, st);
      break;
    case 2: e = run_rescore_g<2>(s, g, kt, q, acand, amin, bounds, idx, keys, block_offset,
                                  fail, err, st);
      break;
    case 4: e = run_rescore_g<4>(s, g, kt, q, acand, amin, bounds, idx, keys, block_offset,
                                  fail, err, st);
      break;
    default: e = run_rescore_g<8>(s, g, kt, q, acand, amin, bounds, idx, keys, block_offset,
                                  fail, err, st);
      break;
  }
  if (e != cudaSuccess) return e;
  // 3. the whole bank, exactly, only if some row failed (the sample's kCand-th bound is
  // a valid start for the 32nd)
  g.run_if = fail;
  if ((e = run_scan<0>(g, mh, ml, kt, q, t0, cand, nullptr, err, st)) != cudaSuccess) return e;
  topk_decode_merge_kernel<<<merge_blocks, 64, 0, st>>>(cand, idx, keys, block_offset, g);
  return cudaGetLastError();
}

}  // namespace msa
