// bsa_internal.h -- the device-side description of one call, shared by the
// host C-ABI (bsa_api.cu) and the kernels.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/bsa.h"

namespace bsa {

constexpr uint16_t kNoBlock = 0xFFFFu;  // unused index slot (BlitzSparseAttention, "sabi")
constexpr int kSlice = 128;             // rows of one q or kv slice (MMA tile height)
constexpr int kSortChunk = 4096;        // keys sorted per CTA before the merge by rank
constexpr uint64_t kAbsentKey = ~0ull;

// status word indices (uint32)
enum : int {
  kStFlags = 0,
  kStFwdNext = 1,   // forward persistent-scheduler counter
  kStFwdItems = 2,
  kStBwdNext = 3,
  kStBwdItems = 4,
  kStTK = 5,        // total kv blocks of this call
  kStNnz = 6,       // inverse-index entries
  kStSumNq = 7,     // query-block rows the lengths need
  kStSubSum = 8,    // (2 words, uint64) sum of the inverse lists' 128-row query slices
  kStWords = 16
};

// per-batch geometry (48 bytes; the layout is mirrored in bsa.h's comment)
struct BatchInfo {
  int32_t qlen, kvlen, nq, nk, qoff, koff;
  int64_t q_tok0, kv_tok0;
  int32_t kvst, pad;  // kvst: kv rows stored for the batch (write bound)
};
static_assert(sizeof(BatchInfo) == 48, "BatchInfo layout");

struct Problem {
  // ---- sizes
  int32_t B, N1, N2, D, g, Hidx, BQ, BKV, W, nsub, ksl;
  int32_t q_layout, kv_layout, dtype;
  int32_t out_dtype;  // dtype of out: dtype, or F16 / BF16 for F8E4M3 inputs
  int64_t Sq, Skv, Tq, Tkv;
  int32_t R;        // index rows per (batch, head) for BNSD; total rows for TND
  int32_t Rg;       // global query-block rows
  int32_t tk_max;   // bound on total kv blocks
  int32_t page_size, max_pages, num_pages;
  int64_t rows_q;   // q storage rows: B*Sq (BNSD) or Tq (TND)
  float scale, scale_log2;  // scale, scale * log2(e)
  int32_t return_lse;
  int32_t causal;  // kv token u visible to query row t iff u <= t + kvlen - qlen
  int32_t deterministic;  // backward: dQ from the q-major pass, no accumulator

  // ---- tensors (strides in elements).  Token row t of batch b, head h:
  //   base + b*sb + (tok0_b + t)*st + h*sh   (tok0 = 0 for BNSD, cu[b] for TND)
  // paged kv: base + page*sb + (u % page)*st + h*sh
  const void *q;  int64_t q_sb, q_sh, q_st;
  const void *k;  int64_t k_sb, k_sh, k_st;
  const void *v;  int64_t v_sb, v_sh, v_st;
  void *out;      int64_t o_sb, o_sh, o_st;
  float *lse;     int64_t l_sb, l_sh, l_st;
  const void *dout; int64_t do_sb, do_sh, do_st;
  void *dq;       int64_t dq_sb, dq_sh, dq_st;
  void *dk;       int64_t dk_sb, dk_sh, dk_st;
  void *dv;       int64_t dv_sb, dv_sh, dv_st;
  const uint16_t *index; int64_t ix_s0, ix_s1, ix_s2;
  const int64_t *cu_q, *cu_kv;
  const int32_t *seqused_kv;
  const int32_t *block_table; int64_t bt_s0;

  // ---- workspace carve-out
  uint32_t *status;
  BatchInfo *batch;
  int32_t *row_batch;   // [Rg]    batch of each global q-block row, -1 if none
  int32_t *kb_batch;    // [tk_max] batch of each global kv block, -1 if none
  uint16_t *comp;       // [Hidx][Rg][W]
  int32_t *ncomp;       // [Hidx][Rg]
  uint64_t *keys;       // sort keys (slots padded to kSortChunk)
  uint64_t *sorted;     // chunk-sorted keys
  int32_t *fwd_items;   // [N1*Rg*nsub]
  int32_t *inv_cnt;     // [Hidx*tk_max]  per (hi, gk): list length
  int32_t *inv_sub;     // [Hidx*tk_max]  per (hi, gk): 128-row q slices in the list
  int32_t *inv_off;     // [Hidx*tk_max + 1]
  int32_t *inv_list;    // [nnz_max]
  int32_t *bwd_items;   // [N2*tk_max*ksl]
  float *dsum;          // [rows_q][N1] rowsum(dOut o out)
  float *dq_acc;        // [rows_q][N1][D]; absent in the deterministic backward
  int64_t fwd_slots, bwd_slots, fwd_slots_pad, bwd_slots_pad;

  // forward: query heads of a GQA group packed into one 128-row tile (the
  // group shares its index row, Hidx == N2): each tile holds 128 / pack_g
  // query rows of each of the pack_g heads, so every K/V chunk streamed in
  // serves the whole group.  1 = one head per tile.
  int32_t pack_g;
  int32_t fsub;  // forward work items per query block: BQ * pack_g / 128
};

// ---- launchers (each returns the first launch error, cudaSuccess otherwise)
cudaError_t launch_prep_geometry(const Problem &p, cudaStream_t s);
cudaError_t launch_prep_compact(const Problem &p, bool fwd_keys, cudaStream_t s);
cudaError_t launch_sort_items(const Problem &p, int64_t slots_pad, int32_t *items, cudaStream_t s);
cudaError_t launch_prep_inverse(const Problem &p, cudaStream_t s);
cudaError_t launch_fwd_main(const Problem &p, cudaStream_t s);
cudaError_t launch_bwd_pre(const Problem &p, cudaStream_t s);
cudaError_t launch_bwd_main(const Problem &p, cudaStream_t s);
cudaError_t launch_bwd_post(const Problem &p, cudaStream_t s);
cudaError_t launch_dq_main(const Problem &p, cudaStream_t s);

int num_sms();

// clears the event pair bsa_set_main_kernel_events armed for this host
// thread's next call (for entry points that return before reaching bsa_fwd
// or bsa_bwd, which consume it)
void drop_pending_events();

}  // namespace bsa
