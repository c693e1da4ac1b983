// Steps 2+3 on the tensor cores (causal prefill, d = 128): block scores and top-k.
//
// One CTA = 128 consecutive tokens of one (sequence, group).  The group-summed queries
// (fp32 sum of the group's heads) are split into bf16 hi + lo planes (x ~ hi + lo to
// ~2^-17 relative) and kept in shared memory; the pooled keys' hi/lo planes stream in
// 128-block chunks through a 2-stage TMA ring.  Each chunk's scores
//     S = Qhi Khi^T + Qhi Klo^T + Qlo Khi^T      (24 tcgen05.mma, M=128 N=128 K=16)
// accumulate in fp32 in one of two TMEM buffers, so the MMAs of chunk c+1 run while the
// four epilogue warps fold chunk c into per-row top lists held in registers.  The list
// is kept sorted (score descending, earlier = lower block index first on ties) with a
// branch-free insertion network; candidates at or below the current last entry are
// rejected with one compare.  The score matrix never leaves the SM.
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
constexpr int kThreads = 192;                // warps 0-3 epilogue, 4 issuer, 5 idle
constexpr uint32_t kHalf = 16384;            // 128 rows x 128 B

struct __align__(8) TBars {
  uint64_t kb_full[2], kb_empty[2], acc_full[2], acc_empty[2], q_full;
  uint32_t tmem_base;
  int abort;
};

struct TopkGeom {
  int64_t S, nb, block;
  int hq, hkv, G, topk;
};

template <int KP>
__device__ __forceinline__ void list_insert(float (&ls)[KP], int (&lj)[KP], float s, int j) {
  // ls descending; strict compares keep the earlier (lower index) entry first on ties.
#pragma unroll
  for (int e = KP - 1; e > 0; --e) {
    const bool up = s > ls[e - 1];
    const bool here = s > ls[e];
    const float ns = up ? ls[e - 1] : (here ? s : ls[e]);
    const int nj = up ? lj[e - 1] : (here ? j : lj[e]);
    ls[e] = ns;
    lj[e] = nj;
  }
  if (s > ls[0]) { ls[0] = s; lj[0] = j; }
}

template <int KP>
__global__ void __launch_bounds__(kThreads, 1)
topk_tc_kernel(const __grid_constant__ CUtensorMap tmHi, const __grid_constant__ CUtensorMap tmLo,
               const __nv_bfloat16* __restrict__ q, int32_t* __restrict__ idx, int* err,
               TopkGeom g) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* Qhi = base;                     // 2 halves
  unsigned char* Qlo = base + 2 * kHalf;
  unsigned char* KB = base + 4 * kHalf;          // stage s: hi halves, lo halves (64 KB)
  TBars* bars = reinterpret_cast<TBars*>(KB + 2 * 4 * kHalf);

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
  if (warp == 0) { tmem_alloc(&bars->tmem_base, 256); tmem_relinquish(); }
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
        unsigned char* dst = KB + st * 4 * kHalf;
        mbar_arrive_expect_tx(&bars->kb_full[st], 4 * kHalf);
        for (int hf = 0; hf < 2; ++hf) {
          const int x = gg * kD + hf * 64;
          tma_load_2d(dst + hf * kHalf, &tmHi, &bars->kb_full[st], x, y_base + c * kChunk);
          tma_load_2d(dst + (2 + hf) * kHalf, &tmLo, &bars->kb_full[st], x, y_base + c * kChunk);
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
        const uint32_t kh = smem_u32(KB + st * 4 * kHalf), kl = kh + 2 * kHalf;
        const uint32_t acc = tmem + st * kChunk;
        int n_mma = 0;
        for (int pass = 0; pass < 3; ++pass) {
          const uint32_t a = pass == 2 ? ql : qh;
          const uint32_t bb = pass == 1 ? kl : kh;
          for (int s = 0; s < kD / 16; ++s) {
            const uint32_t off = (uint32_t)(s >> 2) * kHalf + (uint32_t)(s & 3) * 32;
            umma_ss(acc, sdesc_sw128(a + off, 16, 1024), sdesc_sw128(bb + off, 16, 1024), idS,
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
      const __nv_bfloat16* qr = q + ((b * g.S + (valid ? t : 0)) * g.hq + (int64_t)gg * g.G) * kD;
#pragma unroll 1
      for (int c = 0; c < 16; ++c) {                 // 16 chunks of 8 dims
        float acc8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (valid) {
          for (int h = 0; h < g.G; ++h) {
            float f[8];
            Vec16<__nv_bfloat16>::unpack(ldg16(qr + (int64_t)h * kD + c * 8), f);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc8[e] += f[e];
          }
        }
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          const uint32_t hp = pack_bf16x2(acc8[e], acc8[e + 1]);
          const float h0 = bf16lo_to_f32(hp), h1 = bf16hi_to_f32(hp);
          hw[e / 2] = hp;
          lw[e / 2] = pack_bf16x2(acc8[e] - h0, acc8[e + 1] - h1);
        }
        const uint32_t off = (c >> 3) * kHalf + r * 128 + (((c & 7) ^ (r & 7)) << 4);
        *reinterpret_cast<uint4*>(Qhi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(Qlo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars->q_full);
    }
    const int64_t own = valid ? t / g.block : 0;
    const int n_take = (int)(own < (int64_t)g.topk - 1 ? own : (int64_t)g.topk - 1);
    float ls[KP];
    int lj[KP];
#pragma unroll
    for (int e = 0; e < KP; ++e) { ls[e] = -CUDART_INF_F; lj[e] = -1; }
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    for (int c = 0; c < nch; ++c) {
      const int st = c & 1;
      if (!mbar_wait(&bars->acc_full[st], (c >> 1) & 1)) { fail(); break; }
      tc_fence_after();
      uint32_t sv[4][32];
#pragma unroll
      for (int qd = 0; qd < 4; ++qd) tmem_ld32(lane_base + st * kChunk + qd * 32, sv[qd]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars->acc_empty[st]);
      const int64_t j0 = (int64_t)c * kChunk;
      const int64_t rem = own - j0;
      const int lim = rem <= 0 ? 0 : (rem >= kChunk ? kChunk : (int)rem);
#pragma unroll
      for (int qd = 0; qd < 4; ++qd)
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float s = __uint_as_float(sv[qd][k]);
          if (qd * 32 + k < lim && s > ls[KP - 1]) list_insert<KP>(ls, lj, s, (int)(j0 + qd * 32 + k));
        }
    }
    if (valid) {
      // the n_take best past blocks plus the own block, ascending, -1 padded
      int sel[KP + 1];
      int n = 0;
#pragma unroll
      for (int e = 0; e < KP; ++e)
        if (e < n_take) sel[n++] = lj[e];
      sel[n++] = (int)own;
      for (int a = 1; a < n; ++a) {
        const int x = sel[a];
        int c = a - 1;
        while (c >= 0 && sel[c] > x) { sel[c + 1] = sel[c]; --c; }
        sel[c + 1] = x;
      }
      int32_t* out = idx + ((b * g.hkv + gg) * g.S + t) * (int64_t)g.topk;
      for (int e = 0; e < g.topk; ++e) out[e] = e < n ? sel[e] : -1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}


template <int KP>
cudaError_t run_topk_tc(const Shape& s, const CUtensorMap& mh, const CUtensorMap& ml,
                        const void* q, int32_t* idx, int* err, cudaStream_t st) {
  const size_t smem = 1024 + 12 * (size_t)kHalf + sizeof(TBars);
  cudaError_t e = cudaFuncSetAttribute(topk_tc_kernel<KP>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  TopkGeom g{s.seq, s.nb, s.block, (int)s.hq, (int)s.hkv, (int)(s.hq / s.hkv), (int)s.topk};
  dim3 grid((unsigned)((s.seq + kRows - 1) / kRows), (unsigned)s.hkv, (unsigned)s.batch);
  topk_tc_kernel<KP><<<grid, kThreads, smem, st>>>(mh, ml, (const __nv_bfloat16*)q, idx, err, g);
  return cudaGetLastError();
}

}  // namespace

bool tc_topk_supported(const Shape& s) {
  if (s.dtype != MSA_BF16 || s.d != kD) return false;
  const int64_t G = s.hq / s.hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return false;
  if (s.topk - 1 > 32) return false;
  if (s.batch * s.nb >= ((int64_t)1 << 31) - kChunk) return false;
  return true;
}

cudaError_t launch_topk_prefill_tc(const Shape& s, const void* q, const void* kbar_hi,
                                   const void* kbar_lo, int32_t* idx, int* err, cudaStream_t st) {
  CUtensorMap mh, ml;
  if (!make_bf16_2d_map(&mh, kbar_hi, s.batch * s.nb, s.hkv * kD, kChunk) ||
      !make_bf16_2d_map(&ml, kbar_lo, s.batch * s.nb, s.hkv * kD, kChunk))
    return cudaErrorInvalidValue;
  if (s.topk - 1 <= 16) return run_topk_tc<16>(s, mh, ml, q, idx, err, st);
  return run_topk_tc<32>(s, mh, ml, q, idx, err, st);
}

}  // namespace msa
