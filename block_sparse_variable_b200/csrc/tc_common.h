// tc_common.h -- TMA tensor maps for the tcgen05 kernels (host side).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "bsa_internal.h"

namespace bsa {

// Whole 128-row tiles of the q / k / v tensors in one copy: 5-D maps
// {64 columns, rows, D/64 column halves, heads, batch or page} with box
// {64, 128, D/64, 1, 1}, landing as D/64 consecutive 128-byte-swizzled
// 128-row x 64-column boxes.  Coordinates (0, row, 0, head, batch/page):
//   q, BNSD/TND kv:  rows = token rows (TND: batch coordinate 0)
//   PA_BBND kv:      rows = rows of the page, last coordinate = the page
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

// the q-major dQ pass of the deterministic backward streams Q and dOut with
// the q-tensor box and K, V with the kv box
struct DqMaps {
  CUtensorMap q, k, v, dout;
};

cudaError_t make_dq_maps(const Problem &p, DqMaps &m);

}  // namespace bsa
