// Diagnostic entry point: the two exponentials the attention softmax uses,
// evaluated on caller data, so that their accuracy can be checked on the
// device that runs them (see minf_selftest_exp2 in include/minf.h).
#include "minf_device.cuh"
#include "minf_internal.h"

namespace minf {

__global__ void selftest_exp2_kernel(const float* x, float* y_poly, float* y_mufu, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x0 = x[i], x1 = (i + 1 < n) ? x[i + 1] : 0.f;
  float p0, p1;
  exp2_poly_x2(x0, x1, p0, p1);
  y_poly[i] = p0;
  y_mufu[i] = fast_exp2(x0);
  if (i + 1 < n) {
    y_poly[i + 1] = p1;
    y_mufu[i + 1] = fast_exp2(x1);
  }
}

}  // namespace minf

extern "C" minf_status minf_selftest_exp2(const float* x, float* y_poly, float* y_mufu, int n, void* stream) {
  if (!x || !y_poly || !y_mufu || n < 1) return MINF_ERR_INVALID_ARG;
  const int pairs = (n + 1) / 2;
  minf::selftest_exp2_kernel<<<(pairs + 255) / 256, 256, 0, (cudaStream_t)stream>>>(x, y_poly, y_mufu, n);
  return cudaGetLastError() == cudaSuccess ? MINF_OK : MINF_ERR_CUDA;
}
