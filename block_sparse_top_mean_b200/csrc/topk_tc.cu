// Steps 2+3 on the tensor cores (causal prefill, d = 128): block scores and top-k.
//
// One CTA = 128 consecutive tokens of one (sequence, group).  The group-summed queries
// (fp32 sum of the group's heads) are split into bf16 hi + lo planes (x ~ hi + lo to
// ~2^-17 relative) and kept in shared memory; the pooled keys' hi/lo planes stream in
// 64-block chunks through a 2-stage TMA ring.  Each chunk's scores
//     S = Qhi Khi^T + Qhi Klo^T + Qlo Khi^T      (24 tcgen05.mma, M=128 N=64 K=16)
// accumulate in fp32 in one of two TMEM buffers, so the MMAs of chunk c+1 run while the
// four epilogue warps fold chunk c into the rows' top lists.  Each warp owns 32 token
// rows (its TMEM lanes); it copies their scores to shared memory and then walks them
// row by row with the whole warp: lane l holds entry l of every row's list, sorted by
// (score desc, block index asc), so a candidate is one ballot against the row's
// threshold (entry k-1) and an insertion is a ballot, a popcount and two shuffles.
// Candidates are inserted in ascending block order, which keeps ties on the lower
// index.  The score matrix never leaves the SM.
#include <cudaTypedefs.h>
#include <math_constants.h>

#include "common.cuh"
#include "sm100.cuh"

namespace msa {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kRows = 128;
constexpr int kChunk = 64;                   // pooled keys per MMA chunk (N)
constexpr int kSPad = kChunk + 1;            // row stride of the score copy (no conflicts)
constexpr int kThreads = 192;                // warps 0-3 epilogue, 4 issuer, 5 idle
constexpr uint32_t kHalf = 16384;            // 128 rows x 128 B (query planes)
constexpr uint32_t kKHalf = 8192;            // 64 rows x 128 B (pooled-key planes)

struct __align__(8) TBars {
  uint64_t kb_full[2], kb_empty[2], acc_full[2], acc_empty[2], q_full;
  uint32_t tmem_base;
  int abort;
};

struct TopkGeom {
  int64_t S, nb, block;
  int hq, hkv, G, topk;
};

template <int G>
__global__ void __launch_bounds__(kThreads, 1)
topk_tc_kernel(const __grid_constant__ CUtensorMap tmHi, const __grid_constant__ CUtensorMap tmLo,
               const __nv_bfloat16* __restrict__ q, int32_t* __restrict__ idx, int* err,
               TopkGeom g) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* Qhi = base;                     // 2 halves
  unsigned char* Qlo = base + 2 * kHalf;
  unsigned char* KB = base + 4 * kHalf;          // stage s: hi halves, lo halves (32 KB)
  float* sbuf = reinterpret_cast<float*>(KB + 2 * 4 * kKHalf);     // [kRows][kSPad]
  TBars* bars = reinterpret_cast<TBars*>(sbuf + kRows * kSPad);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int64_t n_tiles_t = (g.S + kRows - 1) / kRows;
  const int64_t tile = n_tiles_t - 1 - blockIdx.x;          // heaviest tiles first
  const int gg = blockIdx.y;
  const int64_t b = blockIdx.z;
  const int64_t t0 = tile * kRows;
  const int64_t t_last = min(t0 + kRows, g.S) - 1;
  const int64_t jmax = t_last / g.block;                    // eligible blocks: j < jmax
  const int nch = (int)((jmax + kChunk - 1) / kChunk);

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->kb_full[s], 1);
      mbar_init(&bars->kb_empty[s], 1);
      mbar_init(&bars->acc_full[s], 1);
      mbar_init(&bars->acc_empty[s], 128);
    }
    mbar_init(&bars->q_full, 128);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) { tmem_alloc(&bars->tmem_base, 128); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort;
  auto fail = [&]() { set_device_error(err, MSA_DEVERR_TIMEOUT); *abort_flag = 1; };

  if (warp == 4) {
    if (lane == 0 && nch > 0) {
      prefetch_tmap(&tmHi);
      prefetch_tmap(&tmLo);
      const uint32_t idS = idesc_bf16(128, kChunk, 0, 0);
      const int y_base = (int)(b * g.nb);
      auto load = [&](int c) {
        const int st = c & 1;
        unsigned char* dst = KB + st * 4 * kKHalf;
        mbar_arrive_expect_tx(&bars->kb_full[st], 4 * kKHalf);
        for (int hf = 0; hf < 2; ++hf) {
          const int x = gg * kD + hf * 64;
          tma_load_2d(dst + hf * kKHalf, &tmHi, &bars->kb_full[st], x, y_base + c * kChunk);
          tma_load_2d(dst + (2 + hf) * kKHalf, &tmLo, &bars->kb_full[st], x, y_base + c * kChunk);
        }
      };
      load(0);
      if (!mbar_wait(&bars->q_full, 0)) fail();
      for (int c = 0; c < nch && !*abort_flag; ++c) {
        const int st = c & 1;
        if (c + 1 < nch) {
          if (c >= 1 && !mbar_wait(&bars->kb_empty[(c + 1) & 1], ((c - 1) >> 1) & 1)) { fail(); break; }
          load(c + 1);
        }
        if (!mbar_wait(&bars->kb_full[st], (c >> 1) & 1)) { fail(); break; }
        if (c >= 2 && !mbar_wait(&bars->acc_empty[st], ((c >> 1) - 1) & 1)) { fail(); break; }
        tc_fence_after();
        const uint32_t qh = smem_u32(Qhi), ql = smem_u32(Qlo);
        const uint32_t kh = smem_u32(KB + st * 4 * kKHalf), kl = kh + 2 * kKHalf;
        const uint32_t acc = tmem + st * kChunk;
        int n_mma = 0;
        for (int pass = 0; pass < 3; ++pass) {
          const uint32_t a = pass == 2 ? ql : qh;
          const uint32_t bb = pass == 1 ? kl : kh;
          for (int s = 0; s < kD / 16; ++s) {
            const uint32_t ko = (uint32_t)(s & 3) * 32;
            umma_ss(acc, sdesc_sw128(a + (uint32_t)(s >> 2) * kHalf + ko, 16, 1024),
                    sdesc_sw128(bb + (uint32_t)(s >> 2) * kKHalf + ko, 16, 1024), idS,
                    n_mma++ > 0);
          }
        }
        umma_commit(&bars->acc_full[st]);
        umma_commit(&bars->kb_empty[st]);
      }
    }
  } else if (warp < 4) {
    // ---------------------------------------------------------------- epilogue rows
    const int r = tid;
    const int64_t t = t0 + r;
    const bool valid = t < g.S;
    // group-summed query row -> bf16 hi/lo planes in the K-major swizzled layout
    {
      const __nv_bfloat16* qr = q + ((b * g.S + (valid ? t : 0)) * g.hq + (int64_t)gg * G) * kD;
#pragma unroll 1
      for (int c0 = 0; c0 < 16; c0 += 4) {         // 4 chunks of 8 dims, loads in flight
        uint4 raw[4][G];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int h = 0; h < G; ++h)
            raw[u][h] = valid ? ldg16(qr + (int64_t)h * kD + (c0 + u) * 8) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = c0 + u;
          float acc8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int h = 0; h < G; ++h) {
            float f[8];
            Vec16<__nv_bfloat16>::unpack(raw[u][h], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc8[e] += f[e];
          }
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const uint32_t hp = pack_bf16x2(acc8[e], acc8[e + 1]);
            hw[e / 2] = hp;
            lw[e / 2] = pack_bf16x2(acc8[e] - bf16lo_to_f32(hp), acc8[e + 1] - bf16hi_to_f32(hp));
          }
          const uint32_t off = (c >> 3) * kHalf + r * 128 + (((c & 7) ^ (r & 7)) << 4);
          *reinterpret_cast<uint4*>(Qhi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(Qlo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars->q_full);
    }
    // Lane l keeps entry l of the sorted lists of the warp's 32 rows; K = topk - 1 <= 31
    // entries are kept (lanes >= K hold the next-best values, also sorted).
    const int K = g.topk - 1;
    float ls[32];
    int lj[32];
#pragma unroll
    for (int rr = 0; rr < 32; ++rr) { ls[rr] = -CUDART_INF_F; lj[rr] = -1; }
    const int64_t row0 = t0 + warp * 32;          // first token of this warp's rows
    float* wbuf = sbuf + warp * 32 * kSPad;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    for (int c = 0; c < nch; ++c) {
      const int st = c & 1;
      if (!mbar_wait_warp(&bars->acc_full[st], (c >> 1) & 1)) { fail(); break; }
      tc_fence_after();
      uint32_t sv[2][32];
      tmem_ld32(lane_base + st * kChunk, sv[0]);
      tmem_ld32(lane_base + st * kChunk + 32, sv[1]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars->acc_empty[st]);
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        wbuf[lane * kSPad + k] = __uint_as_float(sv[0][k]);
        wbuf[lane * kSPad + 32 + k] = __uint_as_float(sv[1][k]);
      }
      __syncwarp();
      const int64_t j0 = (int64_t)c * kChunk;
#pragma unroll
      for (int rr = 0; rr < 32; ++rr) {
        const int64_t tr = row0 + rr;
        const int64_t own_r = tr < g.S ? tr / g.block : 0;
        const int64_t rem = own_r - j0;
        const int lim = K <= 0 ? 0 : (rem <= 0 ? 0 : (rem >= kChunk ? kChunk : (int)rem));
        if (lim == 0) continue;                          // warp-uniform
        const float s0 = wbuf[rr * kSPad + lane];
        const float s1 = wbuf[rr * kSPad + 32 + lane];
        float thr = __shfl_sync(0xffffffffu, ls[rr], K - 1);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const float sh = half ? s1 : s0;
          unsigned m = __ballot_sync(0xffffffffu, sh > thr && half * 32 + lane < lim);
          while (m) {                                    // ascending block index
            const int src = __ffs(m) - 1;
            m &= m - 1;
            const float cs = __shfl_sync(0xffffffffu, sh, src);
            if (!(cs > thr)) continue;                   // threshold rose meanwhile
            const int cj = (int)(j0 + half * 32 + src);
            const int p = __popc(__ballot_sync(0xffffffffu, ls[rr] >= cs));
            const float us = __shfl_up_sync(0xffffffffu, ls[rr], 1);
            const int uj = __shfl_up_sync(0xffffffffu, lj[rr], 1);
            if (lane > p) { ls[rr] = us; lj[rr] = uj; }
            else if (lane == p) { ls[rr] = cs; lj[rr] = cj; }
            thr = __shfl_sync(0xffffffffu, ls[rr], K - 1);
          }
        }
      }
      __syncwarp();
    }
    // Output: the kept past blocks ascending, then the own block, -1 padded.
#pragma unroll 1
    for (int rr = 0; rr < 32; ++rr) {
      const int64_t tr = row0 + rr;
      if (tr >= g.S) break;                              // warp-uniform
      const int64_t own_r = tr / g.block;
      const int n_take = (int)(own_r < K ? own_r : K);
      int key = (lane < n_take) ? lj[rr] : 0x7fffffff;   // bitonic sort, ascending
#pragma unroll
      for (int size = 2; size <= 32; size <<= 1)
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          const int other = __shfl_xor_sync(0xffffffffu, key, stride);
          const bool up = ((lane & size) == 0);
          const bool lower = (lane & stride) == 0;
          key = (lower == up) ? min(key, other) : max(key, other);
        }
      int val = key;
      if (lane == n_take) val = (int)own_r;
      else if (lane > n_take) val = -1;
      if (lane < g.topk)
        idx[((b * g.hkv + gg) * g.S + tr) * (int64_t)g.topk + lane] = val;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}


template <int G>
cudaError_t run_topk_tc(const Shape& s, const CUtensorMap& mh, const CUtensorMap& ml,
                        const void* q, int32_t* idx, int* err, cudaStream_t st) {
  const size_t smem = 1024 + 4 * (size_t)kHalf + 8 * (size_t)kKHalf +
                      (size_t)kRows * kSPad * 4 + sizeof(TBars);
  cudaError_t e = cudaFuncSetAttribute(topk_tc_kernel<G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  TopkGeom g{s.seq, s.nb, s.block, (int)s.hq, (int)s.hkv, (int)(s.hq / s.hkv), (int)s.topk};
  dim3 grid((unsigned)((s.seq + kRows - 1) / kRows), (unsigned)s.hkv, (unsigned)s.batch);
  topk_tc_kernel<G><<<grid, kThreads, smem, st>>>(mh, ml, (const __nv_bfloat16*)q, idx, err, g);
  return cudaGetLastError();
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

cudaError_t launch_topk_prefill_tc(const Shape& s, const void* q, const void* kbar_hi,
                                   const void* kbar_lo, int32_t* idx, int* err, cudaStream_t st) {
  CUtensorMap mh, ml;
  if (!make_bf16_2d_map(&mh, kbar_hi, s.batch * s.nb, s.hkv * kD, kChunk) ||
      !make_bf16_2d_map(&ml, kbar_lo, s.batch * s.nb, s.hkv * kD, kChunk))
    return cudaErrorInvalidValue;
  switch (s.hq / s.hkv) {
    case 1: return run_topk_tc<1>(s, mh, ml, q, idx, err, st);
    case 2: return run_topk_tc<2>(s, mh, ml, q, idx, err, st);
    case 4: return run_topk_tc<4>(s, mh, ml, q, idx, err, st);
    default: return run_topk_tc<8>(s, mh, ml, q, idx, err, st);
  }
}

}  // namespace msa
