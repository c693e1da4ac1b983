// Decode against a memory bank for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or a caching allocator) at the point where they
// run a decode step: a runtime that reserves all device memory up front and forbids
// allocation on its hot path, or a plug-in driven by a host framework that owns every
// allocation and hands it only the tensors of the step.  They still own q, the bank and
// the outputs, but have no workspace to pass.  This entry point runs the same decode
// kernels as msa_decode_fwd with the workspace placed in a file-scope device array of
// fixed size instead.
//
// The array is loaded with the library's device code: every GPU that loads this
// library holds its kMsaDecodeStaticScratch bytes until the process exits.  Host code
// cannot use the array's name as a device address (it names a host-side stand-in), so
// the address is looked up once per device with cudaGetSymbolAddress, on the first call
// made with that device current, and cached.
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kMsaDecodeStaticScratch = MSA_DECODE_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_decode_scratch[kMsaDecodeStaticScratch];

void* g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of g_decode_scratch on the current device (set-up on first use).
msa_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
      return MSA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MSA_OK;
}

}  // namespace

extern "C" msa_status msa_decode_fwd_static(const msa_params* p, int64_t n_query, const void* q,
                                            const float* kbar, const void* kbar_hi,
                                            const void* kbar_lo, const void* k_bank,
                                            const void* v_bank, int32_t* idx, void* o,
                                            float* lse, msa_stream_t stream) {
  // every argument check runs before any CUDA call, with msa_decode_fwd's own statuses
  msa::Shape s;
  bool tc = false, empty = false;
  const msa_status chk = msa::check_decode_args(p, n_query, q, kbar, kbar_hi, kbar_lo, k_bank,
                                                v_bank, idx, o, &s, &tc, &empty);
  if (chk != MSA_OK || empty) return chk;
  if (msa::decode_ws_bytes(s, n_query) > kMsaDecodeStaticScratch)
    return MSA_ERR_WORKSPACE;                                   // beyond the fixed scratch
  void* scratch = nullptr;
  const msa_status st = scratch_address(&scratch);
  if (st != MSA_OK) return st;
  // Only the device error word must start at zero; the rest is written before it is read.
  if (cudaMemsetAsync(scratch, 0, msa::kWsHeader, (cudaStream_t)stream) != cudaSuccess)
    return MSA_ERR_CUDA;
  return msa_decode_fwd(p, n_query, q, kbar, kbar_hi, kbar_lo, k_bank, v_bank, idx, o, lse,
                        scratch, kMsaDecodeStaticScratch, stream);
}

extern "C" msa_status msa_decode_static_read_error(int32_t* bits, msa_stream_t stream) {
  if (bits == nullptr) return MSA_ERR_INVALID_ARG;
  void* scratch = nullptr;
  const msa_status st = scratch_address(&scratch);
  if (st != MSA_OK) return st;
  return msa_read_device_error(scratch, bits, stream);
}
