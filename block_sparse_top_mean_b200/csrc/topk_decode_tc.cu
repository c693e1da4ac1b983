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
constexpr int kAcc = 8;                   // TMEM accumulators of kN columns (all 512)
constexpr int kList = 32;                 // running list length per query (>= topk)
constexpr int kPend = 160;                // pending keys per query: < 32 kept + 128 new
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kThreads = kEpiThreads + 64;   // + TMA producer warp, MMA issuer warp
constexpr int kOwned = kN / kEpiWarps;    // queries per owner warp
constexpr uint32_t kPlane = 16384;        // 128 rows x 128 B: one plane of a half-chunk
constexpr uint32_t kStageBytes = 2 * kPlane;
constexpr uint32_t kQHalf = 8192;         // 64 rows x 128 B: 64 dims of one query plane
constexpr uint32_t kQBytes = 4 * kQHalf;  // hi (2 halves), lo (2 halves)

struct __align__(8) DBars {
  uint64_t full[kStages], empty[kStages], acc_full[kAcc], acc_empty[kAcc], q_full;
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
  int hq, hkv, G, topk, ns_max, ncta_x;
};

constexpr size_t smem_bytes() {
  return 1024 + kQBytes + (size_t)kStages * kStageBytes + (size_t)kN * kPend * 8 +
         (size_t)kN * 8 + sizeof(DBars);
}

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

// GMAX: the sample pass.  Instead of candidate lists the epilogue writes, per query,
// the maximum score of every 32-block group (its order-preserving bits) to gmax
// [query][group][sampled group index].
template <int G, bool GMAX>
__global__ void __launch_bounds__(kThreads, 1)
topk_decode_tc_kernel(const __grid_constant__ CUtensorMap tmHi,
                      const __grid_constant__ CUtensorMap tmLo,
                      const unsigned char* __restrict__ ktiles,
                      const __nv_bfloat16* __restrict__ q, const float* __restrict__ tinit,
                      uint64_t* __restrict__ cand, uint32_t* __restrict__ gmax, int* err,
                      DecGeom g) {
  const int64_t total = (int64_t)g.hkv * g.nch;
  const int64_t u0 = (int64_t)blockIdx.x * g.per;
  const int64_t u1 = u0 + g.per < total ? u0 + g.per : total;
  if (u0 >= u1) return;                          // no units (uniform for the CTA)

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* QI = base;                                   // query planes (B operand)
  unsigned char* KS = QI + kQBytes;                           // stages: hi plane, lo plane
  uint64_t* pend = reinterpret_cast<uint64_t*>(KS + kStages * kStageBytes);   // [kN][kPend]
  int* cnt = reinterpret_cast<int*>(pend + (size_t)kN * kPend);               // [kN]
  float* Ts = reinterpret_cast<float*>(cnt + kN);                             // [kN]
  DBars* bars = reinterpret_cast<DBars*>(Ts + kN);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int64_t qt = blockIdx.y;
  const int nqv = (int)(g.n_query - qt * kN < kN ? g.n_query - qt * kN : kN);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
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
          const int st = (int)(step % kStages);
          if (step >= kStages &&
              !mbar_wait(&bars->empty[st], (uint32_t)((step / kStages) - 1) & 1)) {
            fail();
            break;
          }
          unsigned char* dst = KS + st * kStageBytes;
          mbar_arrive_expect_tx(&bars->full[st], kStageBytes);
          if (tiled) {
            // encoded planes: [plane][group][chunk][half] images of 16 KB each
            const size_t plane = (size_t)g.hkv * g.nch_full * 2 * kPlane;
            const size_t off = (((size_t)gg * g.nch_full + chunk) * 2 + hf) * kPlane;
            bulk_load(dst, ktiles + off, kPlane, &bars->full[st]);
            bulk_load(dst + kPlane, ktiles + plane + off, kPlane, &bars->full[st]);
          } else {
            const int x = gg * kD + hf * 64;
            tma_load_2d(dst, &tmHi, &bars->full[st], x, y);
            tma_load_2d(dst + kPlane, &tmLo, &bars->full[st], x, y);
          }
        }
      }
    }
  } else if (warp == kEpiWarps + 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kM, kN, 0, 0);
      const uint64_t qd = sdesc_sw128(smem_u32(QI), 16, 1024);
      const uint64_t kd0 = sdesc_sw128(smem_u32(KS), 16, 1024);
      int64_t step = 0, tile = 0;
      uint32_t seg = 0;
      for (int64_t u = u0; u < u1 && !*abort_flag; ++u, ++tile) {
        if (u == u0 || u % g.nch == 0) {              // new group: fresh query planes
          if (!mbar_wait(&bars->q_full, seg & 1)) { fail(); break; }
          ++seg;
        }
        const int a = (int)(tile % kAcc);
        if (tile >= kAcc &&
            !mbar_wait(&bars->acc_empty[a], (uint32_t)((tile / kAcc) - 1) & 1)) {
          fail();
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + a * kN;
        bool ok = true;
        for (int hf = 0; hf < 2; ++hf, ++step) {
          const int st = (int)(step % kStages);
          if (!mbar_wait(&bars->full[st], (uint32_t)(step / kStages) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint64_t kh = kd0 + (uint64_t)((st * kStageBytes) >> 4);
          const uint64_t kl = kh + (kPlane >> 4);
          const uint64_t qh = qd + (uint64_t)((hf * kQHalf) >> 4);
          const uint64_t ql = qd + (uint64_t)(((2 + hf) * kQHalf) >> 4);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t o = (uint64_t)(ks * 2);   // 32 bytes per k-step, in 16-B units
            umma_ss(acc, kh + o, qh + o, idesc, (hf | ks) ? 1u : 0u);
            umma_ss(acc, kh + o, ql + o, idesc, 1u);
            umma_ss(acc, kl + o, qh + o, idesc, 1u);
          }
          umma_commit(&bars->empty[st]);
        }
        if (!ok) { fail(); break; }
        umma_commit(&bars->acc_full[a]);
      }
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
      // group-summed query planes of group gg (the previous group's MMAs have all
      // completed: this thread consumed their last accumulator)
#pragma unroll 1
      for (int e = tid; e < kN * 16; e += kEpiThreads) {
        const int n = e >> 4, cc16 = e & 15, hf = cc16 >> 3, cc = cc16 & 7;
        float acc8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (n < nqv) {
          const __nv_bfloat16* qr =
              q + ((qt * kN + n) * (int64_t)g.hq + (int64_t)gg * G) * kD + cc16 * 8;
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
        *reinterpret_cast<uint4*>(QI + hf * kQHalf + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(QI + (2 + hf) * kQHalf + off) =
            make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
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
        const int a = (int)(tile % kAcc);
        if (!aborted && __any_sync(0xffffffffu, *abort_flag != 0)) aborted = true;
        if (!aborted && !mbar_wait_warp(&bars->acc_full[a], (uint32_t)(tile / kAcc) & 1)) {
          fail();
          aborted = true;
        }
        if constexpr (GMAX) {
          if (!aborted) {
            tc_fence_after();
            uint32_t v[32];
            tmem_ld32(lane_base + a * kN, v);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->acc_empty[a]);
            const int64_t j = (u % g.nch) * g.stride * kM + quarter * 32 + lane;
            const bool valid = j < g.nb;
            uint32_t mine = 0u;                   // lane n: group max of query 32*qh + n
#pragma unroll
            for (int n = 0; n < 32; ++n) {
              const uint32_t m = __reduce_max_sync(0xffffffffu, valid ? score_ord(__uint_as_float(v[n])) : 0u);
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
          tmem_ld32(lane_base + a * kN, v);
          tmem_ld_wait();
          const int64_t j = (u % g.nch) * g.stride * kM + quarter * 32 + lane;
          const bool valid = j < g.nb;
          // bit n: this block reaches T of query 32*qh + n
          uint32_t pm = 0u;
#pragma unroll
          for (int n4 = 0; n4 < 8; ++n4) {
            const float4 t4 = *reinterpret_cast<const float4*>(Ts + qh * 32 + n4 * 4);
            pm |= (__uint_as_float(v[n4 * 4 + 0]) >= t4.x ? 1u : 0u) << (n4 * 4 + 0);
            pm |= (__uint_as_float(v[n4 * 4 + 1]) >= t4.y ? 1u : 0u) << (n4 * 4 + 1);
            pm |= (__uint_as_float(v[n4 * 4 + 2]) >= t4.z ? 1u : 0u) << (n4 * 4 + 2);
            pm |= (__uint_as_float(v[n4 * 4 + 3]) >= t4.w ? 1u : 0u) << (n4 * 4 + 3);
          }
          const int nq_here = nqv - qh * 32;       // valid queries of this warp's 32
          if (!valid || nq_here <= 0) pm = 0u;
          else if (nq_here < 32) pm &= (1u << nq_here) - 1u;
          if (__any_sync(0xffffffffu, pm != 0u)) {
            // lane n takes query 32*qh + n: transpose the 32x32 pass matrix (lanes =
            // blocks, bits = queries), reserve that query's slots with one atomic per
            // lane, then every block stores its keys at base + rank among the passes
            uint32_t mt = pm;
#pragma unroll
            for (int sh = 16; sh > 0; sh >>= 1) {
              const uint32_t lo = sh == 16 ? 0x0000ffffu : sh == 8 ? 0x00ff00ffu
                                : sh == 4 ? 0x0f0f0f0fu : sh == 2 ? 0x33333333u : 0x55555555u;
              const uint32_t o = __shfl_xor_sync(0xffffffffu, mt, sh);
              mt = (lane & sh) ? ((mt & ~lo) | ((o >> sh) & lo)) : ((mt & lo) | ((o << sh) & ~lo));
            }
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
              const uint32_t sv = tmem_ld1(lane_base + a * kN + n);
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

// One warp per (query, group): merges the sorted lists of the CTAs that covered the
// group, then writes the best `topk` block indices ascending (-1 padded) or, when `keys`
// is given, the best `topk` keys sorted descending with their block index moved up by
// `block_offset` (a shard's blocks renumbered to bank-wide ids; empty entries stay 0).
__global__ void topk_decode_merge_kernel(const uint64_t* __restrict__ cand,
                                         int32_t* __restrict__ idx, uint64_t* __restrict__ keys,
                                         int64_t block_offset, DecGeom g) {
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
  if (keys != nullptr) {
    if (lane < g.topk) {
      const uint32_t jg = (uint32_t)((int64_t)key_block(y) + block_offset);
      keys[w * g.topk + lane] = y == 0ull ? 0ull : ((y & 0xffffffff00000000ull) | (uint32_t)~jg);
    }
    return;
  }
  // the best topk, ascending by block index (empty entries sort last)
  int j = (lane < g.topk && y != 0ull) ? key_block(y) : 0x7fffffff;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      const int p = __shfl_xor_sync(0xffffffffu, j, jj);
      const bool take_min = ((lane & jj) == 0) == ((lane & k) == 0);
      j = take_min ? min(j, p) : max(j, p);
    }
  }
  if (lane < g.topk) idx[w * g.topk + lane] = j == 0x7fffffff ? -1 : j;
}

// One warp per (query, group): T0 = the 32nd largest of the sampled 32-block group maxima
// (a valid bound: 32 different blocks score at least T0), found bit by bit on the
// order-preserving bits; -inf when fewer than 32 groups were sampled.
constexpr int kThrRegs = 24;                    // register path up to 768 group maxima

__global__ void sample_threshold_kernel(const uint32_t* __restrict__ gmax, float* __restrict__ tout,
                                        int64_t rows, int ngroups) {
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
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
      if (__reduce_add_sync(0xffffffffu, c) >= 32u) prefix = cand;
    }
  } else {
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = prefix | (1u << bit);
      uint32_t c = 0;
      for (int i = lane; i < ngroups; i += 32) c += __ldg(vals + i) >= cand;
      if (__reduce_add_sync(0xffffffffu, c) >= 32u) prefix = cand;
    }
  }
  if (lane == 0) tout[w] = ord_score(prefix);
}

// Sample pass: every kSampleStride-th chunk, when the bank has at least kSampleMinChunks
// chunks per group (the sample then holds >= 16 chunks, 64 block groups, per group).
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

template <int G, bool GMAX>
cudaError_t run_scan(const DecGeom& g, const CUtensorMap& mh, const CUtensorMap& ml,
                     const void* kt, const void* q, const float* tinit, uint64_t* cand,
                     uint32_t* gmax, int* err, cudaStream_t st) {
  const size_t smem = smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(topk_decode_tc_kernel<G, GMAX>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)g.ncta_x, (unsigned)(g.nq_pad / kN));
  topk_decode_tc_kernel<G, GMAX><<<grid, kThreads, smem, st>>>(
      mh, ml, (const unsigned char*)kt, (const __nv_bfloat16*)q, tinit, cand, gmax, err, g);
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
  return true;
}

// Workspace: candidate lists [hkv][CTA slot][query][32] (sized for the larger of the two
// passes), then the sample pass's thresholds [query][hkv].
size_t cand_bytes(const DecGeom& g) {
  return (size_t)g.hkv * g.ns_max * g.nq_pad * kList * sizeof(uint64_t);
}

// Workspace: candidate lists [hkv][CTA slot][query][32], the sample thresholds
// [query][hkv] and the sampled group maxima [query][hkv][group].
struct DecWs {
  size_t cand, tinit, gmax, total;
};
DecWs dec_ws(const Shape& s, int64_t n_query) {
  DecWs w{};
  w.cand = 0;
  w.tinit = (cand_bytes(make_dgeom(s, n_query, 1)) + 255) / 256 * 256;
  w.gmax = w.tinit + ((size_t)n_query * s.hkv * sizeof(float) + 255) / 256 * 256;
  w.total = w.gmax;
  if (use_sample(s)) {
    const DecGeom gs = make_dgeom(s, n_query, kSampleStride);
    w.total += (size_t)n_query * s.hkv * gs.nch * 4 * sizeof(uint32_t);
  }
  return w;
}

size_t topk_decode_tc_ws_bytes(const Shape& s, int64_t n_query) {
  return dec_ws(s, n_query).total;
}

cudaError_t launch_topk_decode_tc(const Shape& s, int64_t n_query, const void* q,
                                  const void* kbar_hi, const void* kbar_lo,
                                  const void* kbar_tiles, int32_t* idx, void* ws, int* err,
                                  cudaStream_t st, uint64_t* keys, int64_t block_offset) {
  CUtensorMap mh{}, ml{};
  if (kbar_tiles == nullptr && (!make_bf16_2d_map(&mh, kbar_hi, s.nb, s.hkv * kD, kM) ||
                                !make_bf16_2d_map(&ml, kbar_lo, s.nb, s.hkv * kD, kM)))
    return cudaErrorInvalidValue;
  const void* kt = kbar_tiles;
  const DecGeom g = make_dgeom(s, n_query, 1);
  const bool sample = use_sample(s);
  const DecWs L = dec_ws(s, n_query);
  char* base = reinterpret_cast<char*>(ws);
  uint64_t* cand = reinterpret_cast<uint64_t*>(base + L.cand);
  float* tinit = reinterpret_cast<float*>(base + L.tinit);
  uint32_t* gmax = reinterpret_cast<uint32_t*>(base + L.gmax);
  cudaError_t e;
  if (sample) {
    // every 8th chunk first: the 32nd largest of its 32-block group maxima per
    // (query, group) is a valid bound that starts the full scan
    const DecGeom gs = make_dgeom(s, n_query, kSampleStride);
    switch (gs.G) {
      case 1: e = run_scan<1, true>(gs, mh, ml, kt, q, nullptr, nullptr, gmax, err, st); break;
      case 2: e = run_scan<2, true>(gs, mh, ml, kt, q, nullptr, nullptr, gmax, err, st); break;
      case 4: e = run_scan<4, true>(gs, mh, ml, kt, q, nullptr, nullptr, gmax, err, st); break;
      default: e = run_scan<8, true>(gs, mh, ml, kt, q, nullptr, nullptr, gmax, err, st); break;
    }
    if (e != cudaSuccess) return e;
    const int64_t rows = n_query * s.hkv;
    // two warps per block: the few hundred warps spread over all SMs
    sample_threshold_kernel<<<(unsigned)((rows + 1) / 2), 64, 0, st>>>(gmax, tinit, rows,
                                                                       (int)(gs.nch * 4));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const float* t0 = sample ? tinit : nullptr;
  switch (g.G) {
    case 1: e = run_scan<1, false>(g, mh, ml, kt, q, t0, cand, nullptr, err, st); break;
    case 2: e = run_scan<2, false>(g, mh, ml, kt, q, t0, cand, nullptr, err, st); break;
    case 4: e = run_scan<4, false>(g, mh, ml, kt, q, t0, cand, nullptr, err, st); break;
    default: e = run_scan<8, false>(g, mh, ml, kt, q, t0, cand, nullptr, err, st); break;
  }
  if (e != cudaSuccess) return e;
  const int64_t warps = n_query * s.hkv;
  topk_decode_merge_kernel<<<(unsigned)((warps + 1) / 2), 64, 0, st>>>(cand, idx, keys,
                                                                        block_offset, g);
  return cudaGetLastError();
}

}  // namespace msa
