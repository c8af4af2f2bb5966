// coalesce.cuh -- coalesced row stores of a warp's accumulator tile.
//
// After a 32x32b TMEM load, thread l of a warp holds C 16-byte chunks of
// row l.  Stored as they are, each warp store instruction writes 16 bytes
// into each of 32 rows: 32 separate lines per instruction, which the memory
// pipeline processes one by one.  An in-register transpose inside groups of
// C lanes (log2 C rounds of xor shuffles, each swapping the off-diagonal
// halves of the group's C x C chunk matrix) leaves lane (g, i) = (l / C,
// l % C) holding chunk i of rows C*g + j in q[j], so that store j writes
// 32/C whole row segments of 16*C contiguous bytes.
#pragma once

#include <stdint.h>

namespace bsa {

template <int C>
__device__ __forceinline__ void transpose_chunks(uint4 (&q)[C], int lane) {
#pragma unroll
  for (int b = C / 2; b >= 1; b >>= 1) {
    const bool hi = (lane & b) != 0;
#pragma unroll
    for (int k = 0; k < C; ++k) {
      if (k & b) continue;
      // lanes without bit b trade their chunk k + b for the partner's chunk k
      const uint4 s = hi ? q[k] : q[k + b];
      uint4 t;
      t.x = __shfl_xor_sync(0xffffffffu, s.x, b);
      t.y = __shfl_xor_sync(0xffffffffu, s.y, b);
      t.z = __shfl_xor_sync(0xffffffffu, s.z, b);
      t.w = __shfl_xor_sync(0xffffffffu, s.w, b);
      if (hi) q[k] = t;
      else q[k + b] = t;
    }
  }
}

// After transpose_chunks: rows 0 .. valid_rows-1 of the warp's 32, row
// pointers row0 + row * row_stride (elements; 16-byte aligned), each row's
// C chunks from its byte 0.  Whole warp.
template <int C, typename T>
__device__ __forceinline__ void store_rows(T *row0, int64_t row_stride, int valid_rows,
                                           const uint4 (&q)[C], int lane) {
  const int g = lane / C, i = lane % C;
#pragma unroll
  for (int j = 0; j < C; ++j) {
    const int row = C * g + j;
    if (row < valid_rows) reinterpret_cast<uint4 *>(row0 + int64_t(row) * row_stride)[i] = q[j];
  }
}

}  // namespace bsa
