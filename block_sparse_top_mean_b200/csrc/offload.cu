// Decode against a bank whose content stays in host memory ("100 Millionen Token:
// Gedaechtnis oder Trugbild?", aitalk.it, section "Das Gehirn mit zwei Geschwindigkeiten":
// the routing keys live in GPU memory, the content keys and values are moved out to the
// CPU's system RAM and transferred to the GPU only once the router selects them; section
// "100 Millionen Token auf 2xA800" puts that transfer on PCIe).
//
// The encoded pooled-key planes are in HBM and the selection runs as usual.  The encoded
// K/V tiles are in pinned host memory, which the GPU reads directly through unified
// addressing.  After the selection, per KV group:
//   mark     flags[g][j] = 1 for every selected block j (any query);
//   scan     one CTA per group numbers the marked blocks in block order: slot[g][j];
//   remap    the selection rewritten as staging slots (ascending like the block ids, so
//            the attention visits the same tiles in the same order), and the list of the
//            staged blocks per group;
//   gather   each staged block's K and V tiles copied from host memory to an HBM staging
//            bank [hkv][n_query * topk blocks][tiles], 16-byte loads, each block fetched
//            once however many queries selected it;
// and the attention of the decode path runs over the staging bank.  The results are
// bitwise those of the decode over an encoded bank held in HBM.
#include "common.cuh"

namespace msa {
namespace {

constexpr int kScanThreads = 1024;

__global__ void offload_mark_kernel(const int32_t* __restrict__ idx, int64_t n_entries, int topk,
                                    int hkv, int64_t nb, uint8_t* __restrict__ flags) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n_entries) return;
  const int j = idx[e];
  if (j < 0 || j >= nb) return;
  const int g = (int)((e / topk) % hkv);
  flags[(int64_t)g * nb + j] = 1;
}

// Exclusive scan of one group's flags: slot[g][j] for marked blocks, count[g].
__global__ void __launch_bounds__(kScanThreads)
offload_scan_kernel(const uint8_t* __restrict__ flags, int64_t nb, int32_t* __restrict__ slot,
                    int32_t* __restrict__ count) {
  __shared__ int s_part[kScanThreads];
  const int g = blockIdx.x;
  const uint8_t* f = flags + (int64_t)g * nb;
  int32_t* sl = slot + (int64_t)g * nb;
  const int64_t per = (nb + kScanThreads - 1) / kScanThreads;
  const int64_t lo = threadIdx.x * per, hi = lo + per < nb ? lo + per : nb;
  int c = 0;
  for (int64_t j = lo; j < hi; ++j) c += f[j];
  s_part[threadIdx.x] = c;
  __syncthreads();
  for (int off = 1; off < kScanThreads; off <<= 1) {     // inclusive Hillis-Steele scan
    const int a = threadIdx.x >= off ? s_part[threadIdx.x - off] : 0;
    __syncthreads();
    s_part[threadIdx.x] += a;
    __syncthreads();
  }
  int base = s_part[threadIdx.x] - c;
  for (int64_t j = lo; j < hi; ++j) {
    sl[j] = f[j] ? base : -1;
    base += f[j];
  }
  if (threadIdx.x == kScanThreads - 1) count[g] = s_part[kScanThreads - 1];
}

__global__ void offload_remap_kernel(const int32_t* __restrict__ idx, int64_t n_entries, int topk,
                                     int hkv, int64_t nb, const int32_t* __restrict__ slot,
                                     int64_t max_slots, int32_t* __restrict__ idx_staged,
                                     int32_t* __restrict__ staged_block) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n_entries) return;
  const int j = idx[e];
  if (j < 0 || j >= nb) { idx_staged[e] = -1; return; }
  const int g = (int)((e / topk) % hkv);
  const int s = slot[(int64_t)g * nb + j];
  idx_staged[e] = s;
  staged_block[(int64_t)g * max_slots + s] = j;        // same value from every query
}

// Copies the staged blocks' K and V tiles from host memory: one thread per 16 bytes.
__global__ void offload_gather_kernel(const uint4* __restrict__ k_host,
                                      const uint4* __restrict__ v_host,
                                      const int32_t* __restrict__ staged_block,
                                      const int32_t* __restrict__ count, int hkv,
                                      int64_t tiles_host, int64_t max_slots, int tpb,
                                      int64_t chunks_per_tile, uint4* __restrict__ k_stage,
                                      uint4* __restrict__ v_stage) {
  const int64_t per_block = (int64_t)tpb * chunks_per_tile;
  const int64_t total = (int64_t)hkv * max_slots * per_block;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t g = i / (max_slots * per_block);
    const int64_t r = i - g * max_slots * per_block;
    const int64_t s = r / per_block;
    if (s >= count[g]) continue;                       // past this group's staged blocks
    const int64_t within = r - s * per_block;          // tile * chunks + chunk
    const int64_t j = staged_block[g * max_slots + s];
    const int64_t src = (g * tiles_host + j * tpb) * chunks_per_tile + within;
    const int64_t dst = (g * max_slots * tpb + s * tpb) * chunks_per_tile + within;
    k_stage[dst] = k_host[src];
    v_stage[dst] = v_host[src];
  }
}

}  // namespace

size_t offload_ws_bytes(const Shape& s, int64_t n_query, int tile_bytes) {
  const int64_t max_slots = n_query * s.topk;
  const int64_t tpb = s.block / 64;
  size_t n = 0;
  auto add = [&](size_t b) { n += (b + 255) / 256 * 256; };
  add((size_t)s.hkv * s.nb);                                 // flags
  add((size_t)s.hkv * s.nb * 4);                             // slot
  add((size_t)s.hkv * 4);                                    // count
  add((size_t)n_query * s.hkv * s.topk * 4);                 // idx_staged
  add((size_t)s.hkv * max_slots * 4);                        // staged_block
  add((size_t)s.hkv * max_slots * tpb * tile_bytes);         // k staging
  add((size_t)s.hkv * max_slots * tpb * tile_bytes);         // v staging
  return n;
}

cudaError_t launch_offload_stage(const Shape& s, int64_t n_query, const int32_t* idx,
                                 const void* k_host, const void* v_host, int tile_bytes,
                                 char* ws, int32_t** idx_staged_out, void** k_stage_out,
                                 void** v_stage_out, cudaStream_t st) {
  const int64_t max_slots = n_query * s.topk;
  const int tpb = (int)(s.block / 64);
  const int64_t tiles_host = (s.seq + 63) / 64;
  size_t off = 0;
  auto take = [&](size_t b) { char* p = ws + off; off += (b + 255) / 256 * 256; return p; };
  uint8_t* flags = (uint8_t*)take((size_t)s.hkv * s.nb);
  int32_t* slot = (int32_t*)take((size_t)s.hkv * s.nb * 4);
  int32_t* count = (int32_t*)take((size_t)s.hkv * 4);
  int32_t* idx_staged = (int32_t*)take((size_t)n_query * s.hkv * s.topk * 4);
  int32_t* staged_block = (int32_t*)take((size_t)s.hkv * max_slots * 4);
  void* k_stage = take((size_t)s.hkv * max_slots * tpb * tile_bytes);
  void* v_stage = take((size_t)s.hkv * max_slots * tpb * tile_bytes);
  cudaError_t e = cudaMemsetAsync(flags, 0, (size_t)s.hkv * s.nb, st);
  if (e != cudaSuccess) return e;
  const int64_t n_entries = n_query * s.hkv * s.topk;
  const unsigned eg = (unsigned)((n_entries + 255) / 256);
  offload_mark_kernel<<<eg, 256, 0, st>>>(idx, n_entries, (int)s.topk, (int)s.hkv, s.nb, flags);
  offload_scan_kernel<<<(unsigned)s.hkv, kScanThreads, 0, st>>>(flags, s.nb, slot, count);
  offload_remap_kernel<<<eg, 256, 0, st>>>(idx, n_entries, (int)s.topk, (int)s.hkv, s.nb, slot,
                                          max_slots, idx_staged, staged_block);
  const int64_t chunks = tile_bytes / 16;
  offload_gather_kernel<<<(unsigned)(sm_count() * 8), 256, 0, st>>>(
      (const uint4*)k_host, (const uint4*)v_host, staged_block, count, (int)s.hkv, tiles_host,
      max_slots, tpb, chunks, (uint4*)k_stage, (uint4*)v_stage);
  *idx_staged_out = idx_staged;
  *k_stage_out = k_stage;
  *v_stage_out = v_stage;
  return cudaGetLastError();
}

}  // namespace msa
