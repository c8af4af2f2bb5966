// selftest.cu -- device checks of building blocks the kernels share with no
// test path of their own (not part of the attention path).
#include <cuda_runtime.h>

#include "bsa_internal.h"
#include "exp2_poly.cuh"
#include "ptx_sm80.cuh"

namespace bsa {
namespace {

__global__ void k_exp2_pair(const float *x, float *y_poly, float *y_mufu, int64_t n) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n;
       i += int64_t(gridDim.x) * blockDim.x) {
    const float v = x[i];
    y_poly[i] = exp2_poly(v);
    y_mufu[i] = ex2(v);
  }
}

}  // namespace
}  // namespace bsa

extern "C" bsa_status bsa_selftest_exp2(const float *x, float *y_poly, float *y_mufu, int64_t n,
                                        void *stream) {
  if (n < 0) return BSA_ERR_PARAM_INVALID;
  if (n == 0) return BSA_OK;
  if (!x || !y_poly || !y_mufu) return BSA_ERR_NULLPTR;
  const int64_t blocks = (n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024;
  bsa::k_exp2_pair<<<unsigned(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y_poly,
                                                                                    y_mufu, n);
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_CUDA;
}
