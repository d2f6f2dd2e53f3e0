// Diagnostic entry points: device helpers of the attention kernels evaluated on their own, so
// that tests can hold them against CUDA's functions and their stated error bounds.
#include "tc_ptx.cuh"

namespace lsrm {
namespace {

// y[i] = poly_exp2_pair applied to x[i] (elements taken two at a time, as the kernels do)
__global__ void diag_exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, long long n) {
  const long long i = 2 * ((long long)blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x0 = x[i];
  const float x1 = i + 1 < n ? x[i + 1] : x0;
  float r0, r1;
  tc::poly_exp2_pair(r0, r1, x0, x1);
  y[i] = r0;
  if (i + 1 < n) y[i + 1] = r1;
}

}  // namespace
}  // namespace lsrm

extern "C" lsrm_status lsrm_diag_exp2_poly(const float* x, float* y, int64_t n, void* stream) {
  if (n < 0 || (n > 0 && (x == nullptr || y == nullptr))) return LSRM_ERR_INVALID_ARG;
  if (n == 0) return LSRM_OK;
  const long long pairs = (n + 1) / 2;
  const unsigned blocks = (unsigned)((pairs + 255) / 256);
  lsrm::diag_exp2_poly_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(x, y, (long long)n);
  return cudaGetLastError() == cudaSuccess ? LSRM_OK : LSRM_ERR_CUDA;
}
