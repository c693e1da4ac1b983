// Steps 2+3 on the tensor cores (causal prefill, d = 128): block scores and top-k.
//
// One CTA = 128 consecutive tokens of one (sequence, group).  The group-summed queries
// (fp32 sum of the group's heads) are split into bf16 hi + lo planes (x ~ hi + lo to
// ~2^-17 relative) and kept in TMEM as the MMA's A operand; the pooled keys' hi/lo
// planes stream in 128-block chunks through a 2-stage TMA ring.  Each chunk's scores
//     S = Qhi Khi^T + Qhi Klo^T + Qlo Khi^T      (24 tcgen05.mma, M=128 N=128 K=16)
// accumulate in fp32 in one of two TMEM buffers, so the MMAs of chunk c+1 run while the
// eight epilogue warps process chunk c: warp w reads TMEM lanes 32*(w%4).. (its token
// rows) and columns 64*(w/4).. of the chunk, so each row is served by two threads.
//
// Selection is exact and takes two passes over the chunks (the MMAs are cheap):
//   pass 1: each thread keeps, in registers, the k-1 largest maxima of groups of 4
//           consecutive scores of its columns (branch-free min/max insertions); the two
//           threads of a row then merge their lists.  The (k-1)-th of the union, T, is
//           a lower bound of the row's (k-1)-th score: k-1 different groups each hold a
//           score >= T.
//   pass 2: the scores are recomputed and every eligible score >= T is appended to the
//           row's buffer in shared memory (about k entries for long rows).
// The row's k-1 best buffered blocks by (score desc, block index asc) are then picked
// exactly.  A row whose buffer would overflow (only degenerate inputs, e.g. exact ties)
// flags its 64-token tile, which the fp32 SIMT selection then recomputes.
// The score matrix never leaves the SM.
#include <cudaTypedefs.h>
#include <math_constants.h>

#include "common.cuh"
#include "sm100.cuh"

namespace msa {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kRows = 128;
constexpr int kChunk = 128;                  // pooled keys per MMA chunk (N)
constexpr int kGroup = 4;                    // scores per group maximum in pass 1
constexpr int kCap = 32;                     // candidate buffer per row and column half
constexpr int kFlagTile = 64;                // tokens per fallback flag
constexpr int kEpiThreads = 256;             // epilogue warps 0-7
constexpr int kThreads = 288;                // warps 0-7 epilogue, 8 issuer
constexpr uint32_t kKHalf = 16384;           // 128 rows x 128 B (pooled-key planes)

constexpr int kStages = 2;                   // pooled-key TMA ring depth

struct __align__(8) TBars {
  uint64_t kb_full[kStages], kb_empty[kStages], acc_full[2], acc_empty[2], q_full;
  uint32_t tmem_base;
  int abort;
};

struct TopkGeom {
  int64_t S, nb, block;
  int hq, hkv, G, topk;
};

template <int G, int KM>
__global__ void __launch_bounds__(kThreads, 1)
topk_tc_kernel(const __grid_constant__ CUtensorMap tmHi, const __grid_constant__ CUtensorMap tmLo,
               const __nv_bfloat16* __restrict__ q, int32_t* __restrict__ idx,
               uint8_t* __restrict__ flags, int* err, TopkGeom g) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* KB = base;                      // stage s: hi halves, lo halves (32 KB)
  float* cand_s = reinterpret_cast<float*>(KB + kStages * 4 * kKHalf);   // [2][kCap][kRows]
  int* cand_j = reinterpret_cast<int*>(cand_s + 2 * kCap * kRows);      // [2][kCap][kRows]
  // the pass-1 lists are exchanged through the candidate area before pass 2 fills it
  float* xl = cand_s;                                                    // [2][KM][kRows]
  int* xcnt = reinterpret_cast<int*>(cand_j + 2 * kCap * kRows);        // [2][kRows]
  TBars* bars = reinterpret_cast<TBars*>(xcnt + 2 * kRows);
  static_assert(2 * KM <= 2 * kCap, "pass-1 lists must fit the candidate area");

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int64_t n_tiles_t = (g.S + kRows - 1) / kRows;
  const int64_t tile = n_tiles_t - 1 - blockIdx.x;          // heaviest tiles first
  const int gg = blockIdx.y;
  const int64_t b = blockIdx.z;
  const int64_t t0 = tile * kRows;
  const int64_t t_last = min(t0 + kRows, g.S) - 1;
  const int64_t jmax = t_last / g.block;                    // eligible blocks: j < jmax
  const int nch = g.topk > 1 ? (int)((jmax + kChunk - 1) / kChunk) : 0;
  const int nsteps = 2 * nch;                               // pass 1 then pass 2

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kb_full[s], 1);
      mbar_init(&bars->kb_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->acc_full[s], 1);
      mbar_init(&bars->acc_empty[s], kEpiThreads);
    }
    mbar_init(&bars->q_full, kEpiThreads);
    bars->abort = 0;
    fence_mbar_init();
  }
  // TMEM: accumulators [0,256), Qhi [256,320), Qlo [320,384) (bf16 pairs per column)
  if (warp == 0) { tmem_alloc(&bars->tmem_base, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort;
  auto fail = [&]() { set_device_error(err, MSA_DEVERR_TIMEOUT); *abort_flag = 1; };

  if (warp == 8) {
    if (lane == 0 && nch > 0) {
      prefetch_tmap(&tmHi);
      prefetch_tmap(&tmLo);
      const uint32_t idS = idesc_bf16(128, kChunk, 0, 0);
      const int y_base = (int)(b * g.nb);
      auto load = [&](int c) {                       // step c streams chunk c mod nch
        const int st = c % kStages;
        unsigned char* dst = KB + st * 4 * kKHalf;
        const int y = y_base + (c % nch) * kChunk;
        mbar_arrive_expect_tx(&bars->kb_full[st], 4 * kKHalf);
        for (int hf = 0; hf < 2; ++hf) {
          const int x = gg * kD + hf * 64;
          tma_load_2d(dst + hf * kKHalf, &tmHi, &bars->kb_full[st], x, y);
          tma_load_2d(dst + (2 + hf) * kKHalf, &tmLo, &bars->kb_full[st], x, y);
        }
      };
      for (int c = 0; c < nsteps && c < kStages; ++c) load(c);
      if (!mbar_wait(&bars->q_full, 0)) fail();
      const uint64_t kdesc0 = sdesc_sw128(smem_u32(KB), 16, 1024);
      constexpr uint64_t kStageStep = (4 * kKHalf) >> 4;
      for (int c = 0; c < nsteps && !*abort_flag; ++c) {
        const int st = c % kStages;
        // refill the stage chunk c-1 used, kStages-1 chunks ahead
        if (c >= 1 && c - 1 + kStages < nsteps) {
          const int ps = (c - 1) % kStages;
          if (!mbar_wait(&bars->kb_empty[ps], ((c - 1) / kStages) & 1)) { fail(); break; }
          load(c - 1 + kStages);
        }
        if (!mbar_wait(&bars->kb_full[st], (c / kStages) & 1)) { fail(); break; }
        if (c >= 2 && !mbar_wait(&bars->acc_empty[c & 1], ((c >> 1) - 1) & 1)) { fail(); break; }
        tc_fence_after();
        const uint64_t kh = kdesc0 + (uint64_t)st * kStageStep;
        const uint64_t kl = kh + ((2 * kKHalf) >> 4);
        const uint32_t acc = tmem + (c & 1) * kChunk;
        // passes: Qhi.Khi, Qhi.Klo, Qlo.Khi (A from TMEM, 8 columns per k-step)
#pragma unroll
        for (int pass = 0; pass < 3; ++pass) {
          const uint32_t a = tmem + (pass == 2 ? 320 : 256);
          const uint64_t bb = pass == 1 ? kl : kh;
#pragma unroll
          for (int s = 0; s < kD / 16; ++s)
            umma_ts(acc, a + s * 8, bb + (uint64_t)((s >> 2) * (kKHalf >> 4) + (s & 3) * 2), idS,
                    (pass > 0 || s > 0) ? 1u : 0u);
        }
        umma_commit(&bars->acc_full[c & 1]);
        umma_commit(&bars->kb_empty[st]);
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue rows
    const int half = warp >> 2;                     // which 32 columns of each chunk
    const int r = (warp & 3) * 32 + lane;           // token row = TMEM lane
    const int64_t t = t0 + r;
    const bool valid = t < g.S;
    // group-summed query row -> bf16 hi/lo pairs in TMEM (this thread: dims 64*half .. +64,
    // i.e. columns 32*half .. +32 of each plane, lane = row)
    {
      const __nv_bfloat16* qr = q + ((b * g.S + (valid ? t : 0)) * g.hq + (int64_t)gg * G) * kD;
      uint32_t hw[32], lw[32];
#pragma unroll
      for (int c0 = 0; c0 < 8; c0 += 4) {           // 4 chunks of 8 dims in flight
        uint4 raw[4][G];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int h = 0; h < G; ++h)
            raw[u][h] = valid ? ldg16(qr + (int64_t)h * kD + (half * 8 + c0 + u) * 8)
                              : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float acc8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int h = 0; h < G; ++h) {
            float f[8];
            Vec16<__nv_bfloat16>::unpack(raw[u][h], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc8[e] += f[e];
          }
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const uint32_t hp = pack_bf16x2(acc8[e], acc8[e + 1]);
            hw[(c0 + u) * 4 + e / 2] = hp;
            lw[(c0 + u) * 4 + e / 2] =
                pack_bf16x2(acc8[e] - bf16lo_to_f32(hp), acc8[e + 1] - bf16hi_to_f32(hp));
          }
        }
      }
      const uint32_t qlane = tmem + ((uint32_t)((warp & 3) * 32) << 16) + half * 32;
      tmem_st32(qlane + 256, hw);
      tmem_st32(qlane + 320, lw);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->q_full);
    }
    const int K = g.topk - 1;                       // past blocks to select
    const int own = valid ? (int)(t / g.block) : 0;
    const int n_take = own < K ? own : K;
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16) + half * 64;
    // pass-1 list of group maxima (this thread's columns), descending; entries >= K spare
    float gm[KM];
#pragma unroll
    for (int e = 0; e < KM; ++e) gm[e] = -CUDART_INF_F;
    float T = -CUDART_INF_F;
    int cnt = 0;
    bool overflow = false;
    float* my_s = cand_s + half * kCap * kRows;
    int* my_j = cand_j + half * kCap * kRows;
    // After a failed wait a warp skips its remaining work but still passes both named
    // barriers below, so the eight epilogue warps always meet at them.
    bool aborted = false;
    for (int c = 0; c < nsteps; ++c) {
      const int st = c & 1;
      const bool pass2 = c >= nch;
      if (c == nch) {
        // threshold for pass 2: the K-th largest of the row's two lists
#pragma unroll
        for (int e = 0; e < KM; ++e) xl[(half * KM + e) * kRows + r] = gm[e];
        asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
        int i0 = 0, i1 = 0;
        for (int e = 0; e < K; ++e) {
          const float a = i0 < KM ? xl[i0 * kRows + r] : -CUDART_INF_F;
          const float bb = i1 < KM ? xl[(KM + i1) * kRows + r] : -CUDART_INF_F;
          if (a >= bb) { T = a; ++i0; } else { T = bb; ++i1; }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
      }
      if (aborted || __any_sync(0xffffffffu, *abort_flag != 0)) {
        aborted = true;
        continue;
      }
      if (!mbar_wait_warp(&bars->acc_full[st], (c >> 1) & 1)) {
        fail();
        aborted = true;
        continue;
      }
      tc_fence_after();
      uint32_t sv[2][32];
      tmem_ld32(lane_base + st * kChunk, sv[0]);
      tmem_ld32(lane_base + st * kChunk + 32, sv[1]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars->acc_empty[st]);
      const int j0 = (pass2 ? c - nch : c) * kChunk + half * 64;
      const int rem = own - j0;
      const int lim = rem <= 0 ? 0 : (rem >= 64 ? 64 : rem);
      if (!pass2) {
        // the 16 group maxima of these 64 columns, sorted (bitonic network), then merged
        // into the descending list: max against the reversed batch, then a bitonic merge
        constexpr int kNG = 64 / kGroup;
        float v[kNG];
#pragma unroll
        for (int q4 = 0; q4 < kNG; ++q4) {
          v[q4] = -CUDART_INF_F;
#pragma unroll
          for (int u = 0; u < kGroup; ++u) {
            const int k = q4 * kGroup + u;
            if (k < lim) v[q4] = fmaxf(v[q4], __uint_as_float(sv[k >> 5][k & 31]));
          }
        }
#pragma unroll
        for (int kk = 2; kk <= kNG; kk <<= 1)
#pragma unroll
          for (int jj = kk >> 1; jj > 0; jj >>= 1)
#pragma unroll
            for (int i = 0; i < kNG; ++i) {
              const int o = i ^ jj;
              if (o > i) {
                const float a = v[i], bq = v[o];
                const bool desc = (i & kk) == 0;
                v[i] = desc ? fmaxf(a, bq) : fminf(a, bq);
                v[o] = desc ? fminf(a, bq) : fmaxf(a, bq);
              }
            }
#pragma unroll
        for (int e = 0; e < KM; ++e)
          if (KM - 1 - e < kNG) gm[e] = fmaxf(gm[e], v[KM - 1 - e]);
#pragma unroll
        for (int jj = KM >> 1; jj > 0; jj >>= 1)
#pragma unroll
          for (int i = 0; i < KM; ++i) {
            const int o = i ^ jj;
            if (o > i) {
              const float a = gm[i], bq = gm[o];
              gm[i] = fmaxf(a, bq);
              gm[o] = fminf(a, bq);
            }
          }
      } else {
#pragma unroll
        for (int k = 0; k < 64; ++k) {
          const float sc = __uint_as_float(sv[k >> 5][k & 31]);
          if (k < lim && sc >= T) {
            if (cnt < kCap) {
              my_s[cnt * kRows + r] = sc;
              my_j[cnt * kRows + r] = j0 + k;
              ++cnt;
            } else {
              overflow = true;
            }
          }
        }
      }
    }
    xcnt[half * kRows + r] = (overflow || aborted) ? -1 : cnt;
    asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
    if (half == 0 && valid) {
      const int c0 = xcnt[r], c1 = xcnt[kRows + r];
      if (c0 < 0 || c1 < 0) {
        flags[(b * g.hkv + gg) * ((g.S + kFlagTile - 1) / kFlagTile) + t / kFlagTile] = 1;
      } else {
        // exact: the n_take best of both halves by (score desc, block index asc)
        int sel[33];
        int n = 0;
        const int tot = c0 + c1;
        for (int e = 0; e < n_take; ++e) {
          int best = -1;
          float bs = 0.f;
          int bj = 0x7fffffff;
          for (int x = 0; x < tot; ++x) {
            const int at = (x < c0 ? x : kCap + x - c0) * kRows + r;
            const int xj = cand_j[at];
            if (xj < 0) continue;                      // taken
            const float xs = cand_s[at];
            if (best < 0 || xs > bs || (xs == bs && xj < bj)) { best = at; bs = xs; bj = xj; }
          }
          if (best < 0) break;
          cand_j[best] = -1;
          sel[n++] = bj;
        }
        sel[n++] = own;
        for (int a2 = 1; a2 < n; ++a2) {
          const int x = sel[a2];
          int c2 = a2 - 1;
          while (c2 >= 0 && sel[c2] > x) { sel[c2 + 1] = sel[c2]; --c2; }
          sel[c2 + 1] = x;
        }
        int32_t* out = idx + ((b * g.hkv + gg) * g.S + t) * (int64_t)g.topk;
        for (int e = 0; e < g.topk; ++e) out[e] = e < n ? sel[e] : -1;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}


template <int G, int KM>
cudaError_t run_topk_tc(const Shape& s, const CUtensorMap& mh, const CUtensorMap& ml,
                        const void* q, int32_t* idx, uint8_t* flags, int* err, cudaStream_t st) {
  const size_t smem = 1024 + (size_t)kStages * 4 * kKHalf + 4 * (size_t)kCap * kRows * 4 +
                      2 * (size_t)kRows * 4 + sizeof(TBars);
  cudaError_t e = cudaFuncSetAttribute(topk_tc_kernel<G, KM>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  TopkGeom g{s.seq, s.nb, s.block, (int)s.hq, (int)s.hkv, (int)(s.hq / s.hkv), (int)s.topk};
  dim3 grid((unsigned)((s.seq + kRows - 1) / kRows), (unsigned)s.hkv, (unsigned)s.batch);
  topk_tc_kernel<G, KM><<<grid, kThreads, smem, st>>>(mh, ml, (const __nv_bfloat16*)q, idx, flags,
                                                      err, g);
  return cudaGetLastError();
}

template <int G>
cudaError_t run_topk_tc_k(const Shape& s, const CUtensorMap& mh, const CUtensorMap& ml,
                          const void* q, int32_t* idx, uint8_t* flags, int* err, cudaStream_t st) {
  if (s.topk - 1 <= 16) return run_topk_tc<G, 16>(s, mh, ml, q, idx, flags, err, st);
  return run_topk_tc<G, 32>(s, mh, ml, q, idx, flags, err, st);
}

}  // namespace

bool tc_topk_supported(const Shape& s) {
  if (s.dtype != MSA_BF16 || s.d != kD) return false;
  const int64_t G = s.hq / s.hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return false;
  if (s.topk > 32) return false;                  // topk - 1 <= 31 list lanes
  if (s.batch * s.nb >= ((int64_t)1 << 31) - kChunk) return false;
  return true;
}

size_t topk_tc_flag_bytes(const Shape& s) {
  return (size_t)s.batch * s.hkv * ((s.seq + kFlagTile - 1) / kFlagTile);
}

cudaError_t launch_topk_prefill_tc(const Shape& s, const void* q, const float* kbar,
                                   const void* kbar_hi, const void* kbar_lo, int32_t* idx,
                                   uint8_t* flags, int* err, cudaStream_t st) {
  CUtensorMap mh, ml;
  if (!make_bf16_2d_map(&mh, kbar_hi, s.batch * s.nb, s.hkv * kD, kChunk) ||
      !make_bf16_2d_map(&ml, kbar_lo, s.batch * s.nb, s.hkv * kD, kChunk))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(flags, 0, topk_tc_flag_bytes(s), st);
  if (e != cudaSuccess) return e;
  switch (s.hq / s.hkv) {
    case 1: e = run_topk_tc_k<1>(s, mh, ml, q, idx, flags, err, st); break;
    case 2: e = run_topk_tc_k<2>(s, mh, ml, q, idx, flags, err, st); break;
    case 4: e = run_topk_tc_k<4>(s, mh, ml, q, idx, flags, err, st); break;
    default: e = run_topk_tc_k<8>(s, mh, ml, q, idx, flags, err, st); break;
  }
  if (e != cudaSuccess) return e;
  // rows whose candidate buffer overflowed: exact fp32 selection of their 64-token tiles
  return launch_topk_prefill_flagged(s, q, kbar, idx, flags, kFlagTile, st);
}

}  // namespace msa
