// selftest.cu -- device checks of building blocks the kernels share with no
// test path of their own (not part of the attention path).
#include <cuda_runtime.h>

#include "bsa_internal.h"
#include "exp2_poly.cuh"
#include "f32x2.cuh"
#include "fp8.cuh"
#include "pack16.cuh"
#include "tc_device.cuh"

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

// One warp waits on an mbarrier that nothing ever arrives at, through the
// same bounded wait the attention kernels use: the wait must give up after
// its time limit, raise BSA_FLAG_TIMEOUT in flags[0] and return, leaving the
// context usable.  Bit 31 would mean the wait wrongly succeeded.
__global__ void k_wait_timeout(uint32_t *flags) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    sm100::mbar_init(b, 1);
    abort_flag = 0;
    sm100::fence_barrier_init();
  }
  __syncthreads();
  const bool ok = wait_warp(b, 0, &abort_flag, flags);
  if (threadIdx.x == 0 && ok) atomicOr(flags + kStFlags, 0x80000000u);
}

// groups of four floats -> one word of four e4m3 bytes, as the FP8 forward
// packs P
__global__ void k_e4m3_pack(const float *x, uint32_t *y, int64_t nwords) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < nwords;
       i += int64_t(gridDim.x) * blockDim.x)
    y[i] = pack_e4m3x4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
}

// the paired fp32 operations the backward's softmax uses, beside their scalar
// forms: out[0..n) fma, [n..2n) add, [2n..3n) mul; pair = f32x2, scalar =
// one rounding per element
__global__ void k_f32x2_pair(const float *a, const float *b, const float *c, float *pair,
                             float *scalar, int64_t n) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; 2 * i < n;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t e = 2 * i;
    const float2 A = make_float2(a[e], a[e + 1]), B = make_float2(b[e], b[e + 1]);
    const float2 C = make_float2(c[e], c[e + 1]);
    const float2 f = fma2(A, B, C), s = add2(A, B), m = mul2(A, B);
    pair[e] = f.x, pair[e + 1] = f.y;
    pair[n + e] = s.x, pair[n + e + 1] = s.y;
    pair[2 * n + e] = m.x, pair[2 * n + e + 1] = m.y;
    scalar[e] = __fmaf_rn(A.x, B.x, C.x), scalar[e + 1] = __fmaf_rn(A.y, B.y, C.y);
    scalar[n + e] = __fadd_rn(A.x, B.x), scalar[n + e + 1] = __fadd_rn(A.y, B.y);
    scalar[2 * n + e] = __fmul_rn(A.x, B.x), scalar[2 * n + e + 1] = __fmul_rn(A.y, B.y);
  }
}

}  // namespace
}  // namespace bsa

extern "C" bsa_status bsa_selftest_wait_timeout(uint32_t *flags, void *stream) {
  if (!flags) return BSA_ERR_NULLPTR;
  bsa::k_wait_timeout<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(flags);
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_CUDA;
}

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

extern "C" bsa_status bsa_selftest_e4m3(const float *x, uint32_t *packed, int64_t n, void *stream) {
  if (n < 0 || n % 4 != 0) return BSA_ERR_PARAM_INVALID;
  if (n == 0) return BSA_OK;
  if (!x || !packed) return BSA_ERR_NULLPTR;
  const int64_t w = n / 4;
  const int64_t blocks = (w + 255) / 256 < 1024 ? (w + 255) / 256 : 1024;
  bsa::k_e4m3_pack<<<unsigned(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(x, packed, w);
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_CUDA;
}

extern "C" bsa_status bsa_selftest_f32x2(const float *a, const float *b, const float *c,
                                         float *pair, float *scalar, int64_t n, void *stream) {
  if (n < 0 || n % 2 != 0) return BSA_ERR_PARAM_INVALID;
  if (n == 0) return BSA_OK;
  if (!a || !b || !c || !pair || !scalar) return BSA_ERR_NULLPTR;
  const int64_t w = n / 2;
  const int64_t blocks = (w + 255) / 256 < 1024 ? (w + 255) / 256 : 1024;
  bsa::k_f32x2_pair<<<unsigned(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(a, b, c, pair,
                                                                                     scalar, n);
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ERR_CUDA;
}
