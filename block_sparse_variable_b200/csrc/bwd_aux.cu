// bwd_aux.cu -- the small kernels around the backward main kernel
// (BlockSparseAttentionGrad README, "Formula"):
//   pre:   softmax_grad = Dsum_t = sum_d dOut[t,d] * out[t,d]  (fp32), and the
//          fp32 dQ accumulator cleared;
//   post:  dq = dtype(scale * dQacc) for every query row, and zeros for the
//          stored kv rows past each batch's used length that no backward work
//          item covers.
#include <cuda_runtime.h>

#include <cmath>

#include "addr.cuh"
#include "bsa_internal.h"
#include "launch.cuh"
#include "pack16.cuh"

namespace bsa {
namespace {


// q storage row r -> (batch, batch-local token) for the q-layout tensors
__device__ __forceinline__ int64_t qstore_off(const Problem &p, int64_t sb, int64_t sh, int64_t st,
                                              int64_t r, int h) {
  if (p.q_layout == BSA_LAYOUT_BNSD) return (r / p.Sq) * sb + (r % p.Sq) * st + int64_t(h) * sh;
  return r * st + int64_t(h) * sh;
}

// eight lanes per (query row, head): each reads 16 bytes of dOut and out per
// pass (a warp covers four (row, head) pairs, 512 bytes of each tensor per
// pass), then the eight partial dot products are summed by shuffles; the
// same lanes zero the pair's row of the fp32 dQ accumulator
template <typename T>
__global__ void k_bwd_pre(const Problem p) {
  griddep_wait();
  griddep_launch_next();
  const int64_t w = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 3;
  const int sub = threadIdx.x & 7;
  const bool live = w < p.rows_q * p.N1;
  float acc = 0.f;
  int64_t r = 0;
  int h = 0;
  if (live) {
    r = w / p.N1;
    h = int(w % p.N1);
    const T *dO = static_cast<const T *>(p.dout) + qstore_off(p, p.do_sb, p.do_sh, p.do_st, r, h);
    const T *O = static_cast<const T *>(p.out) + qstore_off(p, p.o_sb, p.o_sh, p.o_st, r, h);
    for (int d = sub * 8; d < p.D; d += 64) {
      const uint4 a = *reinterpret_cast<const uint4 *>(dO + d);
      const uint4 c = *reinterpret_cast<const uint4 *>(O + d);
      const uint32_t av[4] = {a.x, a.y, a.z, a.w}, cv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 x = Pack2<T>::unpack(av[e]);
        const float2 y = Pack2<T>::unpack(cv[e]);
        acc = fmaf(x.x, y.x, fmaf(x.y, y.y, acc));
      }
    }
    // the pair's fp32 dQ accumulator row starts at zero (the same eight
    // lanes, 16 bytes each per pass)
    if (p.dq_acc) {
      uint4 *acc_row = reinterpret_cast<uint4 *>(p.dq_acc + w * p.D);
      for (int d = sub * 4; d < p.D; d += 32) acc_row[d / 4] = make_uint4(0, 0, 0, 0);
    }
  }
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (live && sub == 0) p.dsum[r * p.N1 + h] = acc;
}

// dq = dtype(scale * dQacc) for every q storage row
template <typename T>
__global__ void k_dq_convert(const Problem p) {
  griddep_wait();
  griddep_launch_next();
  const int64_t n8 = p.rows_q * p.N1 * (p.D / 8);
  const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= n8) return;
  const int64_t e = idx * 8;
  const int d = int(e % p.D);
  const int h = int((e / p.D) % p.N1);
  const int64_t r = e / (int64_t(p.D) * p.N1);
  const float4 x0 = *reinterpret_cast<const float4 *>(p.dq_acc + e);
  const float4 x1 = *reinterpret_cast<const float4 *>(p.dq_acc + e + 4);
  uint4 o;
  o.x = Pack2<T>::pack(x0.x * p.scale, x0.y * p.scale);
  o.y = Pack2<T>::pack(x0.z * p.scale, x0.w * p.scale);
  o.z = Pack2<T>::pack(x1.x * p.scale, x1.y * p.scale);
  o.w = Pack2<T>::pack(x1.z * p.scale, x1.w * p.scale);
  *reinterpret_cast<uint4 *>(static_cast<T *>(p.dq) + qstore_off(p, p.dq_sb, p.dq_sh, p.dq_st, r, h) +
                             d) = o;
}

// zeros for the kv rows of each batch that no backward item covers:
// [round_up(kvlen, 128), kvst) -- stored rows past the used length
template <typename T>
__global__ void k_kv_zero_tail(const Problem p) {
  griddep_wait();
  griddep_launch_next();
  const int b = blockIdx.y;
  const BatchInfo bi = p.batch[b];
  const int lo = ((bi.kvlen + kSlice - 1) / kSlice) * kSlice;
  const int64_t rows = bi.kvst > lo ? bi.kvst - lo : 0;
  const int CH = p.D / 8;
  const int64_t total = rows * p.N2 * CH;
  T *dkg = static_cast<T *>(p.dk);
  T *dvg = static_cast<T *>(p.dv);
  for (int64_t x = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; x < total;
       x += int64_t(gridDim.x) * blockDim.x) {
    const int ch = int(x % CH);
    const int h2 = int((x / CH) % p.N2);
    const int u = lo + int(x / (int64_t(CH) * p.N2));
    int pg = 0;
    if (p.kv_layout == BSA_LAYOUT_PA_BBND) {
      pg = kv_page(p, b, u);
      if (pg < 0) continue;
    }
    const uint4 z = make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4 *>(dkg + kv_row(p, p.dk_sb, p.dk_sh, p.dk_st, bi, b, h2, u, pg) + ch * 8) = z;
    *reinterpret_cast<uint4 *>(dvg + kv_row(p, p.dv_sb, p.dv_sh, p.dv_st, bi, b, h2, u, pg) + ch * 8) = z;
  }
}

}  // namespace

// (the dQ accumulator, absent in the deterministic backward, is zeroed by
// the same kernel)
cudaError_t launch_bwd_pre(const Problem &p, cudaStream_t s) {
  const int64_t pairs = p.rows_q * p.N1;  // eight lanes each
  const unsigned grid = unsigned((pairs * 8 + 255) / 256);
  cudaError_t e = p.dtype == BSA_BF16 ? launch_dep(k_bwd_pre<__nv_bfloat16>, dim3(grid), dim3(256), 0, s, p)
                                      : launch_dep(k_bwd_pre<__half>, dim3(grid), dim3(256), 0, s, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_bwd_post(const Problem &p, cudaStream_t s) {
  const int64_t n8 = p.rows_q * p.N1 * (p.D / 8);
  const unsigned grid = unsigned((n8 + 255) / 256);
  const dim3 zgrid(64, unsigned(p.B));
  cudaError_t e = cudaSuccess;
  if (p.dtype == BSA_BF16) {
    if (p.dq_acc && (e = launch_dep(k_dq_convert<__nv_bfloat16>, dim3(grid), dim3(256), 0, s, p)) != cudaSuccess)
      return e;
    e = launch_dep(k_kv_zero_tail<__nv_bfloat16>, zgrid, dim3(256), 0, s, p);
  } else {
    if (p.dq_acc && (e = launch_dep(k_dq_convert<__half>, dim3(grid), dim3(256), 0, s, p)) != cudaSuccess)
      return e;
    e = launch_dep(k_kv_zero_tail<__half>, zgrid, dim3(256), 0, s, p);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace bsa
