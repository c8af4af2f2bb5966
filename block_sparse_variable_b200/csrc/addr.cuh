// addr.cuh -- token-row addressing shared by the attention kernels.
//   q-like tensors:  base + b*sb + (tok0_b + t)*st + h*sh
//   kv (BNSD/TND):   base + b*sb + (kv_tok0_b + u)*st + h2*sh
//   kv (PA_BBND):    base + page*sb + (u % page_size)*st + h2*sh with
//                    page = block_table[b][u / page_size]
//                    (GenericBlockSparseAttention, "Paged Attention")
#pragma once

#include "bsa_internal.h"

namespace bsa {

// page of kv token u of batch b, or -1 when the table entry is out of range
__device__ __forceinline__ int kv_page(const Problem &p, int b, int u) {
  const int pg = p.block_table[int64_t(b) * p.bt_s0 + u / p.page_size];
  return (pg < 0 || pg >= p.num_pages) ? -1 : pg;
}

// element offset of row u (head h2) given its page (ignored unless paged)
__device__ __forceinline__ int64_t kv_row(const Problem &p, int64_t sb, int64_t sh, int64_t st,
                                          const BatchInfo &bi, int b, int h2, int u, int page) {
  if (p.kv_layout == BSA_LAYOUT_PA_BBND)
    return int64_t(page) * sb + int64_t(u % p.page_size) * st + int64_t(h2) * sh;
  return int64_t(b) * sb + (bi.kv_tok0 + u) * st + int64_t(h2) * sh;
}

__device__ __forceinline__ int64_t q_row(int64_t sb, int64_t sh, int64_t st, const BatchInfo &bi,
                                         int b, int h, int t) {
  return int64_t(b) * sb + (bi.q_tok0 + t) * st + int64_t(h) * sh;
}

}  // namespace bsa
