// tc_common.h -- TMA tensor maps for the tcgen05 kernels (host side).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "bsa_internal.h"

namespace bsa {

// 128-byte-swizzled 64-column x 128-row boxes of the q / k / v tensors.
//   q, BNSD/TND kv:  4-D {D, token rows, heads, batch}
//   PA_BBND kv:      4-D {D, heads, page rows, pages}   (box 64 x 1 x 128 x 1)
struct FwdMaps {
  CUtensorMap q, k, v;
};

cudaError_t make_fwd_maps(const Problem &p, FwdMaps &m);

// the backward also streams dOut with the q-tensor box, and adds its dQ
// tiles into the fp32 accumulator [rows][N1][D] through a 3-D map
// {D, N1, rows} with 32-column x 1-head x 128-row boxes (128-byte swizzle)
struct BwdMaps {
  CUtensorMap q, k, v, dout, dq_acc;
};

cudaError_t make_bwd_maps(const Problem &p, BwdMaps &m);

}  // namespace bsa
