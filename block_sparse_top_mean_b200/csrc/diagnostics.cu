// Diagnostic entry points: evaluate device helpers of the kernels on caller data, so
// tests can hold them to their error bounds on the GPU.
#include "common.cuh"
#include "fastmath.cuh"

namespace {

__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
  const int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x0 = x[i], x1 = i + 1 < n ? x[i + 1] : 0.f;
  float p0, p1;
  msa::fastmath::poly_exp2x2(x0, x1, p0, p1);
  y[i] = p0;
  if (i + 1 < n) y[i + 1] = p1;
}

}  // namespace

extern "C" msa_status msa_exp2_poly_eval(const float* x, float* y, int64_t n,
                                         msa_stream_t stream) {
  if (n < 0) return MSA_ERR_INVALID_ARG;
  if (n == 0) return MSA_OK;
  if (x == nullptr || y == nullptr) return MSA_ERR_INVALID_ARG;
  if (n > ((int64_t)1 << 40)) return MSA_ERR_UNSUPPORTED;
  const int64_t pairs = (n + 1) / 2;
  exp2_poly_kernel<<<(unsigned)((pairs + 255) / 256), 256, 0, (cudaStream_t)stream>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}
