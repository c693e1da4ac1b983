// Step 4 for decode against a bank: exact attention of each (query, group) over its
// selected blocks, streamed through shared memory (bf16, d = 128, block % 64 == 0).
//
// Decode is HBM-bound: every selected K/V byte is read once per (query, group) and the
// arithmetic is ~2 FLOP per byte.  The kernel is shaped around the stream:
//   - persistent CTAs (one per SM) take work units round-robin; a unit is one
//     (query, group) and 8 consecutive selection slots (a split);
//   - a producer warp walks the same unit/slot sequence as the consumers and TMA-loads
//     each selected 64-key tile of K and V (128-byte swizzle, 2 x 8 KB each; with an
//     encoded bank, one 16 KB bulk copy each, see bank_tiles.cu) into a
//     6-stage ring; the first tile of a unit also carries the group's G query rows
//     (one bulk copy); both roles load a unit's selection entries one unit ahead;
//   - four consumer warps split each tile's 64 keys (16 each) and run the contractions
//     on mma.sync m16n8k16 (bf16 in, fp32 accumulate) with the G heads as the M rows
//     (padded to 16): S = Q K^T from ldmatrix'ed K, an online softmax in base 2 per
//     head, P (bf16) reused in registers as the A operand of O += P V with ldmatrix.trans'ed V;
//   - at the end of a unit each warp writes its own normalised partial and log-sum-exp
//     (no cross-warp merge, no barrier); combine_splits_kernel merges the 4 x nsplit
//     partials of a (query, group).
#include <cudaTypedefs.h>
#include <math_constants.h>

#include "common.cuh"
#include "sm100.cuh"

namespace msa {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kTileKeys = 64;               // keys per stage (one TMA box of rows)
constexpr int kStages = 6;
constexpr int kConsumers = 4;               // warps 0-3
constexpr int kThreads = 32 * kConsumers + 32;   // + producer warp 4
constexpr int kSlotsPerUnit = 8;            // selection slots per work unit (a split)
constexpr uint32_t kHalfBytes = kTileKeys * 128;        // 64 keys x 64 dims (bf16)
constexpr uint32_t kKVBytes = 4 * kHalfBytes;           // K halves, V halves (32 KB)
constexpr uint32_t kQBytesMax = 8 * kD * 2;             // up to 8 heads of one group
constexpr uint32_t kStageStride = kKVBytes + 2048;      // 1024-aligned (34 KB)
static_assert(kKVBytes + kQBytesMax <= kStageStride, "query rows must fit the stage");
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct __align__(8) ABars {
  uint64_t full[kStages], empty[kStages];
  int abort;
};

struct DecAttnGeom {
  int64_t S, nb, block, n_rows;   // bank tokens, bank blocks, block size, n_query * hkv
  int64_t ntiles;                 // 64-key tiles per head of an encoded bank
  int hq, hkv, topk, nsplit, tiles_per_block;
  float scale_log2;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                          uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// C[16x8] += A[16x16] B[16x8], bf16 inputs, fp32 accumulators (rows g, g+8; cols 2t, 2t+1).
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The kSlotsPerUnit selection entries of unit u (-1 beyond topk), one vector load when
// the row is 16-byte aligned.
struct Slots {
  int4 a, b;
};
__device__ __forceinline__ int4 load4(const int32_t* p, int s0, int topk) {
  if ((topk & 3) == 0 && s0 + 4 <= topk) return __ldg(reinterpret_cast<const int4*>(p));
  int4 r;
  r.x = s0 + 0 < topk ? __ldg(p + 0) : -1;
  r.y = s0 + 1 < topk ? __ldg(p + 1) : -1;
  r.z = s0 + 2 < topk ? __ldg(p + 2) : -1;
  r.w = s0 + 3 < topk ? __ldg(p + 3) : -1;
  return r;
}
__device__ __forceinline__ Slots unit_slots(const int32_t* __restrict__ idx, int64_t u,
                                            const DecAttnGeom& g) {
  const int64_t row = u / g.nsplit;
  const int s0 = (int)(u % g.nsplit) * kSlotsPerUnit;
  const int32_t* p = idx + row * g.topk + s0;
  Slots r;
  r.a = load4(p, s0, g.topk);
  r.b = s0 + 4 < g.topk ? load4(p + 4, s0 + 4, g.topk) : make_int4(-1, -1, -1, -1);
  return r;
}
__device__ __forceinline__ int slot_of(const Slots& v, int i) {
  const int4& h = i < 4 ? v.a : v.b;
  const int k = i & 3;
  return k == 0 ? h.x : k == 1 ? h.y : k == 2 ? h.z : h.w;
}

// Byte offset of 16-byte chunk c (0..15, 8 dims each) of key row r inside a K or V tile.
__device__ __forceinline__ uint32_t tile_off(int r, int c) {
  return (uint32_t)(c >> 3) * kHalfBytes + (uint32_t)r * 128u + ((uint32_t)((c & 7) ^ (r & 7)) << 4);
}

// Both roles walk the same sequence: units blockIdx.x, +gridDim.x, ...; in each, the
// unit's slots in order, skipping -1 and out-of-range entries (the producer flags the
// latter), and every 64-key tile of a selected block that starts inside the bank.
template <int G>
__global__ void __launch_bounds__(kThreads, 1)
attn_decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const unsigned char* __restrict__ ktiles,
                      const unsigned char* __restrict__ vtiles,
                      const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ idx,
                      float* __restrict__ po, float* __restrict__ plse, int* err, DecAttnGeom g) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  ABars* bars = reinterpret_cast<ABars*>(base + kStages * kStageStride);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], kConsumers);
    }
    bars->abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort_flag = &bars->abort;
  auto fail = [&]() { set_device_error(err, MSA_DEVERR_TIMEOUT); *abort_flag = 1; };
  const int64_t n_units = g.n_rows * g.nsplit;

  if (warp == kConsumers) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const bool tiled = ktiles != nullptr;
      if (!tiled) {
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
      }
      int64_t step = 0;
      Slots nxt{};
      if (blockIdx.x < n_units) nxt = unit_slots(idx, blockIdx.x, g);
      for (int64_t u = blockIdx.x; u < n_units && !*abort_flag; u += gridDim.x) {
        const Slots cur = nxt;                          // the next unit's slots load meanwhile
        if (u + gridDim.x < n_units) nxt = unit_slots(idx, u + gridDim.x, g);
        const int64_t row = u / g.nsplit;
        const int64_t n = row / g.hkv;
        const int gg = (int)(row % g.hkv);
        bool first = true;
        for (int sl = 0; sl < kSlotsPerUnit && !*abort_flag; ++sl) {
          const int64_t j = slot_of(cur, sl);
          if (j == -1) continue;
          if (j < -1 || j >= g.nb) { set_device_error(err, MSA_DEVERR_IDX_RANGE); continue; }
          for (int t = 0; t < g.tiles_per_block; ++t, ++step) {
            const int64_t key0 = j * g.block + (int64_t)t * kTileKeys;
            if (key0 >= g.S) break;
            const int st = (int)(step % kStages);
            if (step >= kStages &&
                !mbar_wait(&bars->empty[st], (uint32_t)((step / kStages) - 1) & 1)) {
              fail();
              break;
            }
            unsigned char* dst = base + st * kStageStride;
            const uint32_t qb = first ? (uint32_t)(G * kD * 2) : 0u;
            mbar_arrive_expect_tx(&bars->full[st], kKVBytes + qb);
            if (tiled) {
              // encoded bank: the (group, 64-key tile) is one contiguous 16 KB image
              const size_t off = ((size_t)gg * g.ntiles + (size_t)(key0 / kTileKeys)) * 2 * kHalfBytes;
              bulk_load(dst, ktiles + off, 2 * kHalfBytes, &bars->full[st]);
              bulk_load(dst + 2 * kHalfBytes, vtiles + off, 2 * kHalfBytes, &bars->full[st]);
            } else {
              for (int hf = 0; hf < 2; ++hf) {
                const int x = gg * kD + hf * 64;
                tma_load_2d(dst + hf * kHalfBytes, &tmK, &bars->full[st], x, (int)key0);
                tma_load_2d(dst + (2 + hf) * kHalfBytes, &tmV, &bars->full[st], x, (int)key0);
              }
            }
            if (first) bulk_load(dst + kKVBytes, q + (n * g.hq + (int64_t)gg * G) * kD, qb,
                                 &bars->full[st]);
            first = false;
          }
        }
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumers (warps 0-3)
  const int gr = lane >> 2, t4 = lane & 3;       // fragment row (head) and column pair
  const float c2 = g.scale_log2;
  int64_t step = 0;
  bool aborted = false;
  Slots nxt{};
  if (blockIdx.x < n_units) nxt = unit_slots(idx, blockIdx.x, g);
  for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x) {
    const Slots cur = nxt;
    if (u + gridDim.x < n_units) nxt = unit_slots(idx, u + gridDim.x, g);
    const int64_t row = u / g.nsplit;
    const int split = (int)(u % g.nsplit);
    float m_run = -CUDART_INF_F, l_run = 0.f;       // head gr (valid when gr < G)
    float o[16][4];
#pragma unroll
    for (int dt = 0; dt < 16; ++dt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[dt][e] = 0.f;
    uint32_t qa[8][2];                              // A fragments of Q (rows gr; +8 rows are 0)
    bool first = true;
    for (int sl = 0; sl < kSlotsPerUnit; ++sl) {
      const int64_t j = slot_of(cur, sl);
      if (j < 0 || j >= g.nb) continue;
      for (int t = 0; t < g.tiles_per_block; ++t, ++step) {
        const int64_t key0 = j * g.block + (int64_t)t * kTileKeys;
        if (key0 >= g.S) break;
        const int st = (int)(step % kStages);
        if (aborted || __any_sync(0xffffffffu, *abort_flag != 0)) { aborted = true; continue; }
        if (!mbar_wait_warp(&bars->full[st], (uint32_t)(step / kStages) & 1)) {
          fail();
          aborted = true;
          continue;
        }
        const unsigned char* stg = base + st * kStageStride;
        const uint32_t sK = smem_u32(stg), sV = sK + 2 * kHalfBytes;
        if (first) {
          const uint32_t* qs = reinterpret_cast<const uint32_t*>(stg + kKVBytes);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            qa[ks][0] = gr < G ? qs[(gr * kD + ks * 16 + 2 * t4) / 2] : 0u;
            qa[ks][1] = gr < G ? qs[(gr * kD + ks * 16 + 8 + 2 * t4) / 2] : 0u;
          }
          first = false;
        }
        // S = Q K^T for this warp's 16 keys (two n-tiles of 8)
        float sc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[nt][e] = 0.f;
        }
        const int mi = lane >> 3, ri = lane & 7;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int kr = warp * 16 + nt * 8 + ri;
#pragma unroll
          for (int ks = 0; ks < 8; ks += 2) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4(sK + tile_off(kr, 2 * ks + (mi & 1) + 2 * (mi >> 1)), b0, b1, b2, b3);
            mma16816(sc[nt], qa[ks][0], 0u, qa[ks][1], 0u, b0, b1);
            mma16816(sc[nt], qa[ks + 1][0], 0u, qa[ks + 1][1], 0u, b2, b3);
          }
        }
        // online softmax of head gr over the 16 keys (columns 2*t4, 2*t4+1 of each n-tile)
        float x[4];
        float mx = -CUDART_INF_F;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int64_t key = key0 + warp * 16 + nt * 8 + 2 * t4 + e;
            const float v = key < g.S ? sc[nt][e] * c2 : -CUDART_INF_F;
            x[nt * 2 + e] = v;
            mx = fmaxf(mx, v);
          }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float m_new = fmaxf(m_run, mx);
        const float m_use = m_new == -CUDART_INF_F ? 0.f : m_new;
        const float alpha = exp2f(m_run - m_use);
        float p[4], ps = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) { p[e] = exp2f(x[e] - m_use); ps += p[e]; }
        l_run = l_run * alpha + ps;
        m_run = m_new;
#pragma unroll
        for (int dt = 0; dt < 16; ++dt) { o[dt][0] *= alpha; o[dt][1] *= alpha; }
        const uint32_t pa0 = pack_bf16x2(p[0], p[1]);      // keys 2t4, 2t4+1
        const uint32_t pa2 = pack_bf16x2(p[2], p[3]);      // keys 8+2t4, 8+2t4+1
        // O += P V (16 n-tiles of 8 dims; V^T fragments by ldmatrix.trans)
        const int vr = warp * 16 + (mi & 1) * 8 + ri;
#pragma unroll
        for (int dt = 0; dt < 16; dt += 2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(sV + tile_off(vr, dt + (mi >> 1)), b0, b1, b2, b3);
          mma16816(o[dt], pa0, 0u, pa2, 0u, b0, b1);
          mma16816(o[dt + 1], pa0, 0u, pa2, 0u, b2, b3);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->empty[st]);
      }
    }
    // this warp's partial over its 16-key slices of the unit's tiles, normalised, with its
    // log-sum-exp: one split of the (query, group) for combine_splits_kernel
    float lsum = l_run;
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
    if (gr < G) {
      const int64_t pi = ((row * g.nsplit + split) * kConsumers + warp) * G + gr;
      const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
      float* dst = po + pi * kD + 2 * t4;
#pragma unroll
      for (int dt = 0; dt < 16; ++dt)
        *reinterpret_cast<float2*>(dst + dt * 8) = make_float2(o[dt][0] * inv, o[dt][1] * inv);
      if (t4 == 0) plse[pi] = lsum > 0.f ? (m_run + log2f(lsum)) * kLn2 : -CUDART_INF_F;
    }
  }
}

size_t smem_bytes() { return 1024 + (size_t)kStages * kStageStride + sizeof(ABars); }

template <int G>
cudaError_t run_dec_attn(const DecAttnGeom& g, const CUtensorMap& mk, const CUtensorMap& mv,
                         const void* kt, const void* vt, const void* q, const int32_t* idx,
                         float* po, float* plse, int* err, cudaStream_t st) {
  const size_t smem = smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(attn_decode_tc_kernel<G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int64_t units = g.n_rows * g.nsplit;
  int grid = sm_count();
  if (units < grid) grid = (int)units;
  attn_decode_tc_kernel<G><<<grid, kThreads, smem, st>>>(
      mk, mv, (const unsigned char*)kt, (const unsigned char*)vt, (const __nv_bfloat16*)q, idx,
      po, plse, err, g);
  return cudaGetLastError();
}

}  // namespace

bool tc_decode_attn_supported(const Shape& s) {
  if (s.dtype != MSA_BF16 || s.d != kD) return false;
  if (s.block % kTileKeys != 0) return false;
  const int64_t G = s.hq / s.hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return false;
  if (s.seq >= ((int64_t)1 << 31) - kTileKeys) return false;    // TMA row coordinate
  return true;
}

int decode_attn_tc_nsplit(const Shape& s) {
  return (int)((s.topk + kSlotsPerUnit - 1) / kSlotsPerUnit);
}
int decode_attn_tc_partials(const Shape& s) { return decode_attn_tc_nsplit(s) * kConsumers; }

cudaError_t launch_attn_decode_tc(const Shape& s, int64_t n_query, const void* q, const void* k,
                                  const void* v, const void* k_tiles, const void* v_tiles,
                                  const int32_t* idx, float* po, float* plse, int* err,
                                  cudaStream_t st) {
  CUtensorMap mk{}, mv{};
  if (k_tiles == nullptr && (!make_bf16_2d_map(&mk, k, s.seq, s.hkv * kD, kTileKeys) ||
                             !make_bf16_2d_map(&mv, v, s.seq, s.hkv * kD, kTileKeys)))
    return cudaErrorInvalidValue;
  DecAttnGeom g{};
  g.ntiles = (s.seq + kTileKeys - 1) / kTileKeys;
  g.S = s.seq; g.nb = s.nb; g.block = s.block; g.n_rows = n_query * s.hkv;
  g.hq = (int)s.hq; g.hkv = (int)s.hkv; g.topk = (int)s.topk;
  g.nsplit = decode_attn_tc_nsplit(s);
  g.tiles_per_block = (int)(s.block / kTileKeys);
  g.scale_log2 = s.scale * kLog2e;
  switch (s.hq / s.hkv) {
    case 1: return run_dec_attn<1>(g, mk, mv, k_tiles, v_tiles, q, idx, po, plse, err, st);
    case 2: return run_dec_attn<2>(g, mk, mv, k_tiles, v_tiles, q, idx, po, plse, err, st);
    case 4: return run_dec_attn<4>(g, mk, mv, k_tiles, v_tiles, q, idx, po, plse, err, st);
    default: return run_dec_attn<8>(g, mk, mv, k_tiles, v_tiles, q, idx, po, plse, err, st);
  }
}

}  // namespace msa
