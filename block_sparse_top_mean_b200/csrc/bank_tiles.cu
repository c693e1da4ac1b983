// Offline encoding of a decode memory bank (bf16, d = 128) into the images the decode
// kernels stream with one bulk copy per tile.
//
// The routing keys of a bank are computed once, when the bank is written; so can its
// memory layout.  In the natural layout [S, hkv, d] one KV head of a 64-key block is
// 64 runs of 256 bytes, 2 KB apart, which a tensor-map copy fetches as 128-byte rows.
// The encoded layout stores, per KV head, each 64-key tile (and each 128-block chunk of
// the pooled-key planes) contiguously and already in the 128-byte-swizzled shared-
// memory layout of a TMA box (16-byte chunk c of row r at position c ^ (r % 8)), so a
// single 1-D bulk copy lands it ready for ldmatrix / tcgen05:
//   K, V tiles   [hkv][ceil(S/64)][2 halves of 64 dims][64 rows][128 B]   16 KB a tile
//   kbar tiles   [2 planes: hi, lo][hkv][ceil(nb/128)][2 halves][128 rows][128 B]
//                then bounds [2][hkv] fp32: max_j ||lo_j||_2 and max_j ||hi_j||_2 per KV
//                head, which bound how far a hi-plane-only score can be from the full one
// Rows past the end of the bank (keys >= S, blocks >= nb) are zero.
#include "common.cuh"

namespace msa {
namespace {

// One thread per 16-byte chunk of the output; reads the matching chunk of the source
// row [row, hkv, 128] (16 chunks per (row, head)).
template <int ROWS>
__global__ void tile_image_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                  int64_t n_rows, int hkv, int64_t n_tiles) {
  const int64_t total = (int64_t)hkv * n_tiles * 2 * ROWS * 8;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int cpos = (int)(e & 7);
    const int r = (int)((e >> 3) % ROWS);
    const int64_t rest = (e >> 3) / ROWS;        // (head * n_tiles + tile) * 2 + half
    const int h = (int)(rest & 1);
    const int64_t tile = (rest >> 1) % n_tiles;
    const int g = (int)((rest >> 1) / n_tiles);
    const int c = cpos ^ (r & 7);
    const int64_t row = tile * ROWS + r;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (row < n_rows) v = src[(row * hkv + g) * 16 + h * 8 + c];
    dst[e] = v;
  }
}

template <int ROWS>
cudaError_t launch_image(const void* src, void* dst, int64_t n_rows, int hkv, cudaStream_t st) {
  const int64_t n_tiles = (n_rows + ROWS - 1) / ROWS;
  const int64_t total = (int64_t)hkv * n_tiles * 2 * ROWS * 8;
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = (int64_t)sm_count() * 16;
  if (blocks > cap) blocks = cap;
  tile_image_kernel<ROWS><<<(unsigned)blocks, 256, 0, st>>>(
      (const uint4*)src, (uint4*)dst, n_rows, hkv, n_tiles);
  return cudaGetLastError();
}

// One warp per (block, KV head): the Euclidean norms of the block's hi and lo rows,
// folded into the per-head maxima with an unsigned atomic max (non-negative floats order
// like their bit patterns; the bounds start at zero).
__global__ void plane_bounds_kernel(const __nv_bfloat16* __restrict__ hi,
                                    const __nv_bfloat16* __restrict__ lo, int64_t n_rows,
                                    int hkv, unsigned* __restrict__ bounds) {
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (w >= n_rows) return;                     // n_rows = nb * hkv, row w = (j, head)
  const int g = (int)(w % hkv);
  const uint2 h = *reinterpret_cast<const uint2*>(hi + w * 128 + lane * 4);
  const uint2 l = *reinterpret_cast<const uint2*>(lo + w * 128 + lane * 4);
  float sh = 0.f, sl = 0.f;
  const uint32_t hw[2] = {h.x, h.y}, lw[2] = {l.x, l.y};
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const float a = __uint_as_float(hw[k] << 16), b = __uint_as_float(hw[k] & 0xffff0000u);
    const float c = __uint_as_float(lw[k] << 16), d = __uint_as_float(lw[k] & 0xffff0000u);
    sh += a * a + b * b;
    sl += c * c + d * d;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sh += __shfl_xor_sync(0xffffffffu, sh, o);
    sl += __shfl_xor_sync(0xffffffffu, sl, o);
  }
  if (lane == 0) {
    atomicMax(bounds + g, __float_as_uint(sqrtf(sl)));
    atomicMax(bounds + hkv + g, __float_as_uint(sqrtf(sh)));
  }
}

}  // namespace

size_t bank_kv_tiles_bytes(const Shape& s) {
  return (size_t)s.hkv * ((s.seq + 63) / 64) * 16384;
}
size_t bank_kbar_planes_bytes(const Shape& s) {
  return (size_t)s.hkv * ((s.nb + 127) / 128) * 32768;
}
size_t bank_kbar_tiles_bytes(const Shape& s) { return 2 * bank_kbar_planes_bytes(s) + 256; }

cudaError_t launch_encode_bank(const Shape& s, const void* k, const void* v, const void* kbar_hi,
                               const void* kbar_lo, void* k_tiles, void* v_tiles,
                               void* kbar_tiles, cudaStream_t st) {
  cudaError_t e = cudaSuccess;
  if (k_tiles != nullptr && (e = launch_image<64>(k, k_tiles, s.seq, (int)s.hkv, st)) != cudaSuccess)
    return e;
  if (v_tiles != nullptr && (e = launch_image<64>(v, v_tiles, s.seq, (int)s.hkv, st)) != cudaSuccess)
    return e;
  if (kbar_tiles != nullptr) {
    char* hi_img = reinterpret_cast<char*>(kbar_tiles);
    char* lo_img = hi_img + bank_kbar_planes_bytes(s);
    char* bounds = lo_img + bank_kbar_planes_bytes(s);
    if ((e = launch_image<128>(kbar_hi, hi_img, s.nb, (int)s.hkv, st)) != cudaSuccess) return e;
    if ((e = launch_image<128>(kbar_lo, lo_img, s.nb, (int)s.hkv, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(bounds, 0, 256, st)) != cudaSuccess) return e;
    const int64_t rows = s.nb * s.hkv;
    if (rows > 0) {
      plane_bounds_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
          (const __nv_bfloat16*)kbar_hi, (const __nv_bfloat16*)kbar_lo, rows, (int)s.hkv,
          (unsigned*)bounds);
    }
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace msa
