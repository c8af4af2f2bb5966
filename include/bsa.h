/*
 * bsa.h -- C ABI of the B200 (sm_100a) block-sparse variable-length
 * FlashAttention library (libbsa.so).
 *
 * The operation (BlockSparseAttentionGrad README, "Formula"; GenericBlock-
 * SparseAttention article, "sparse attention mechanism"):
 *
 *     out = softmax(scale * Q * K_sparse^T) * V_sparse
 *
 * where query block i (BQ rows) attends only to the KV blocks (BKV rows)
 * listed in its row of a uint16 block index (BlitzSparseAttention article,
 * "sabi" section: ascending batch-local KV block ids, unused slots 0xFFFF).
 * The forward pass also returns the per-row natural-log log-sum-exp of the
 * scaled scores (same article, "softmax_lse output"; its all-ones example
 * fixes lse = ln S + sqrt(D) for S keys and D = head dim at scale 1/sqrt(D)).
 * The backward pass (BlockSparseAttentionGrad README, "Formula") recomputes
 * P from the LSE and returns dQ, dK, dV:
 *     softmax_grad = rowsum(dOut o out), dP = dOut V^T,
 *     dS = P o (dP - softmax_grad), dV = P^T dOut,
 *     dQ = dS K scale, dK = dS^T Q scale.
 *
 * API shape: two calls per pass, as in the aclnn two-phase interface
 * (aclnnFlashAttentionUnpaddingScoreGradV2 article, sections 3 and 5): a
 * *_get_workspace call validates every descriptor and returns the scratch
 * size, then the exec call runs on a CUDA stream.  There is no executor
 * object: the library is stateless and every argument is passed again.
 *
 * Ownership: the caller owns every buffer, including the workspace (device
 * memory, at least the returned size, 256-byte aligned).  The library
 * allocates nothing and keeps no state between calls.  One workspace must
 * not be used by two calls that may overlap on the GPU.
 *
 * Errors: every entry point returns a bsa_status and never aborts.  Host
 * validation covers shapes, strides, dtypes, layouts and attributes; the
 * *values* of cu_seqlens, seqused_kv, the index and the block table are not
 * read on the host (GenericBlockSparseAttention article, "values are not
 * checked at tiling").  The device skips invalid values and records them as
 * BSA_FLAG_* bits in the workspace status word, read with bsa_read_status;
 * no invalid value is used as an address.  The readings (the pages leave
 * them open):
 *   - a cu_seqlens pair that decreases, starts below 0 or ends past its
 *     tensor, or a seqused_kv below 0 or above the stored kv length, counts
 *     as length 0 (BAD_SEQLEN): a query batch without rows, a kv batch
 *     nothing can select (its index entries are then out of range:
 *     BAD_INDEX).  Batches whose ranges overlap (possible only with a
 *     decreasing cu_seqlens) give unspecified results for the shared rows;
 *   - a block-table entry outside [0, num_pages) that covers a used kv token
 *     raises BAD_PAGE, whether or not a row selects it; the tokens it covers
 *     take no part, and the backward writes no dk/dv for them;
 *   - a TND query block with no index row (fewer rows than the lengths need)
 *     selects nothing (BAD_INDEX): out 0, lse -inf, dq 0.
 * Rows of the q-layout tensors that belong to no batch (past the last
 * batch, or of a batch whose cu_seqlens_q pair is invalid) are not written
 * by the forward; the default backward writes dq 0 there.
 */
#ifndef BSA_H_
#define BSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------- tensors */
enum {
  BSA_F16 = 1,
  BSA_BF16 = 2,
  BSA_F32 = 3,
  BSA_U16 = 4,
  BSA_I32 = 5,
  BSA_I64 = 6,
  BSA_F8E4M3 = 7  /* OCP 8-bit float E4M3 (forward q/k/v only) */
};

/* A strided view of device memory.  data == NULL (or a NULL descriptor
 * pointer) means "absent" for optional arguments.  Strides are in elements;
 * the last dimension must be contiguous (stride 1). */
typedef struct bsa_tensor {
  void *data;
  int32_t dtype;
  int32_t ndim;
  int64_t shape[4];
  int64_t stride[4];
} bsa_tensor;

/* Layouts (BlockSparseAttentionGrad README, "layouts"; GenericBlockSparse-
 * Attention article, "Paged Attention"):
 *   BNSD     q [B, N1, Sq, D],  kv [B, N2, Skv, D]
 *   TND      q [Tq, N1, D],     kv [Tkv, N2, D]; batch b is rows
 *            cu_seqlens[b] .. cu_seqlens[b+1]-1
 *   PA_BBND  kv only: [num_pages, page_size, N2, D]; kv token u of batch b
 *            is page block_table[b][u / page_size], row u % page_size. */
enum { BSA_LAYOUT_BNSD = 0, BSA_LAYOUT_TND = 1, BSA_LAYOUT_PA_BBND = 2 };

typedef struct bsa_params {
  int32_t q_layout;       /* BSA_LAYOUT_BNSD or BSA_LAYOUT_TND */
  int32_t kv_layout;      /* BNSD (needs q BNSD), TND, or PA_BBND (needs q TND) */
  int64_t num_heads;      /* N1 */
  int64_t num_kv_heads;   /* N2; 0 means N1.  N1 % N2 == 0 (GQA) */
  int64_t block_shape[2]; /* {BQ, BKV}, each in {128, 256, 512, 1024} */
  double scale;           /* 0 means 1/sqrt(D) */
  int32_t return_lse;     /* forward only: write lse when non-zero */
  int32_t mask_type;      /* BSA_MASK_NONE or BSA_MASK_CAUSAL */
  int32_t deterministic;  /* backward only: non-zero for bitwise reproducible
                             dq (see bsa_bwd); forward: ignored */
} bsa_params;

/* Token mask inside the selected blocks (GenericBlockSparseAttention article,
 * mask section: a built-in causal mode).  BSA_MASK_CAUSAL keeps kv token u for
 * query row t of batch b only when u <= t + kvlen_b - qlen_b: the mask is
 * aligned to the end of the kv sequence (the page does not state the
 * alignment; this is our reading, the usual one when a query chunk continues
 * a longer kv sequence).  A row that keeps no token gives out 0, lse -inf. */
enum { BSA_MASK_NONE = 0, BSA_MASK_CAUSAL = 1 };

/* Status codes: the first three echo the aclnn codes the pages list
 * (161001 null pointer, 161002 invalid parameter, 561103 inner error). */
typedef enum bsa_status {
  BSA_OK = 0,
  BSA_ERR_NULLPTR = 161001,       /* a required pointer or descriptor is NULL */
  BSA_ERR_PARAM_INVALID = 161002, /* shapes / strides / dtypes / attributes disagree */
  BSA_ERR_UNSUPPORTED = 161003,   /* valid request outside what this library supports */
  BSA_ERR_WORKSPACE = 161004,     /* workspace NULL, misaligned or too small */
  BSA_ERR_CUDA = 561000,          /* a kernel launch or CUDA call failed */
  BSA_ERR_INNER = 561103          /* internal inconsistency */
} bsa_status;

/* Bits of the device status word (bsa_read_status). */
#define BSA_FLAG_BAD_INDEX 0x1u   /* an index entry >= ceil(kvlen/BKV) or not above the
                                     previous accepted entry (skipped), or more query
                                     blocks than index rows (TND) */
#define BSA_FLAG_BAD_SEQLEN 0x2u  /* cu_seqlens / seqused_kv contradict the storage
                                     (that length counts as 0) */
#define BSA_FLAG_BAD_PAGE 0x4u    /* a block-table entry outside [0, num_pages) covers
                                     a used kv token (its tokens take no part) */
#define BSA_FLAG_TIMEOUT 0x8u     /* a bounded device wait gave up (pipeline fault) */
#define BSA_FLAG_INTERNAL 0x10u   /* a kernel precondition failed (internal error) */

/* ------------------------------------------------------------- forward */
/* Arguments:
 *   q       BNSD [B,N1,Sq,D] or TND [Tq,N1,D], F16 or BF16, D in {64, 128};
 *           or F8E4M3 with D = 128 (see below)
 *   k, v    BNSD [B,N2,Skv,D], TND [Tkv,N2,D] or PA_BBND [P,page,N2,D];
 *           same dtype as q; page % 128 == 0
 *   index   U16. BNSD q: [B, Hidx, ceil(Sq/BQ), W]; TND q: [Hidx, R, W] with
 *           the rows of batch b after the ceil(qlen/BQ) rows of every earlier
 *           batch.  Hidx == N1 (own row per q head) or N2 (the group of q
 *           heads sharing a kv head shares the row).  Entries are batch-local
 *           kv block ids; 0xFFFF = unused slot.
 *   cu_seqlens_q   I64 [B+1], required for TND q (prefix sums, [0] == 0)
 *   cu_seqlens_kv  I64 [B+1], required for TND kv, absent otherwise
 *   seqused_kv     I32 [B], optional; required for PA_BBND.  kv tokens at or
 *                  past seqused_kv[b] are ignored.
 *   block_table    I32 [B, max_pages], required for PA_BBND
 *   out     same shape/dtype as q (written for every query row of every
 *           batch; rows with no selected key get 0); F16 or BF16 for F8E4M3
 *           inputs, and then its dtype is the output type
 *   lse     F32, BNSD [B,N1,Sq] / TND [Tq,N1]; required when return_lse
 *           (rows with no selected key get -inf)
 * FP8 inputs (GenericBlockSparseAttention article, quantization table,
 * quantType 5): q, k, v in E4M3 without scale tensors; the scores are exact
 * e4m3 products summed in fp32, and P is cast to E4M3 (round to nearest
 * even, saturating) before the P V product, while the row sums l and lse
 * come from the unrounded fp32 P.  Each output element then lies within
 * sum_u (2^-4 P_u + 2^-10) |v_u| / l of the exact result (P_u relative to
 * the row maximum), plus the output's own rounding.  Strides of FP8
 * tensors are multiples of 16 elements.  The backward takes 16-bit inputs
 * only (BSA_ERR_UNSUPPORTED for E4M3).
 */
bsa_status bsa_fwd_get_workspace(const bsa_tensor *q, const bsa_tensor *k, const bsa_tensor *v,
                                 const bsa_tensor *index, const bsa_tensor *cu_seqlens_q,
                                 const bsa_tensor *cu_seqlens_kv, const bsa_tensor *seqused_kv,
                                 const bsa_tensor *block_table, const bsa_params *params,
                                 const bsa_tensor *out, const bsa_tensor *lse,
                                 size_t *workspace_bytes);

/* Same arguments, then the workspace and a cudaStream_t (NULL = legacy
 * default stream).  Asynchronous: returns after the launches. */
bsa_status bsa_fwd(const bsa_tensor *q, const bsa_tensor *k, const bsa_tensor *v,
                   const bsa_tensor *index, const bsa_tensor *cu_seqlens_q,
                   const bsa_tensor *cu_seqlens_kv, const bsa_tensor *seqused_kv,
                   const bsa_tensor *block_table, const bsa_params *params,
                   const bsa_tensor *out, const bsa_tensor *lse, void *workspace,
                   size_t workspace_bytes, void *stream);

/* Forward without a caller-supplied workspace; allocates nothing.
 * (An addition of this library: the pages have no counterpart.)
 *
 * For callers that cannot allocate device memory when they run the
 * forward -- for example a plugin executed by an inference runtime whose
 * contract forbids allocation inside its execute step, or an engine that
 * fixes its device-memory budget at start-up.  Arguments and results are
 * those of bsa_fwd; the caller still passes every input and output.  The
 * scratch lives in a fixed 32 MiB array inside the library that every GPU
 * loading the library keeps until the process exits.
 *   - A problem whose forward workspace (bsa_fwd_get_workspace) exceeds
 *     32 MiB is rejected with BSA_ERR_WORKSPACE before any launch.
 *   - The first call on a device sets the array up there: CUDA places a
 *     module's device data on the GPU when it is first used, so that call
 *     grows device memory by the 32 MiB, then looks the array's address up
 *     and caches it.  Make one call per device at start-up -- before the
 *     phase in which the caller may not allocate, and before any stream
 *     capture on that device; later calls allocate nothing.
 *   - All calls share the one array, which keeps the last call's contents;
 *     each call initialises everything it reads, but two calls that may
 *     overlap on the GPU (different streams, different threads) race and
 *     must be serialised by the caller.
 *   - bsa_read_status cannot see this scratch; the status word is not
 *     available to the caller. */
bsa_status bsa_fwd_static_workspace(const bsa_tensor *q, const bsa_tensor *k, const bsa_tensor *v,
                                    const bsa_tensor *index, const bsa_tensor *cu_seqlens_q,
                                    const bsa_tensor *cu_seqlens_kv,
                                    const bsa_tensor *seqused_kv, const bsa_tensor *block_table,
                                    const bsa_params *params, const bsa_tensor *out,
                                    const bsa_tensor *lse, void *stream);

/* ------------------------------------------------------------ backward */
/* q, k, v, index, cu_seqlens_*, seqused_kv, block_table: as for bsa_fwd.
 *   out, lse  the forward's outputs (lse required)
 *   dout      same shape/dtype as q
 *   dq        same shape/dtype as q; every row written
 *   dk, dv    same shape/dtype as k / v.  Every kv row of every batch is
 *             written (zeros where no query selects it), except that under
 *             PA_BBND only the pages block_table[b][0 .. ceil(kvlen_b/page))
 *             are written; other pages are left untouched.
 * By default dq is summed in fp32 from many CTAs through the L2 (order of
 * the additions varies between runs, so dq may differ in its last bits).
 * With params->deterministic set, dq comes from a separate query-major pass
 * that recomputes P and dS and sums each row's contributions in index order
 * on one SM (the deterministic template of the aclnnFlashAttention-
 * UnpaddingScoreGradV2 article, section 6.1: no two cores add into the same
 * address), so dq, dk and dv are bitwise the same on every run; it costs
 * the q-major pass's extra S and dP products.  The workspace size depends on
 * the flag.
 */
bsa_status bsa_bwd_get_workspace(const bsa_tensor *q, const bsa_tensor *k, const bsa_tensor *v,
                                 const bsa_tensor *out, const bsa_tensor *dout,
                                 const bsa_tensor *lse, const bsa_tensor *index,
                                 const bsa_tensor *cu_seqlens_q, const bsa_tensor *cu_seqlens_kv,
                                 const bsa_tensor *seqused_kv, const bsa_tensor *block_table,
                                 const bsa_params *params, const bsa_tensor *dq,
                                 const bsa_tensor *dk, const bsa_tensor *dv,
                                 size_t *workspace_bytes);

bsa_status bsa_bwd(const bsa_tensor *q, const bsa_tensor *k, const bsa_tensor *v,
                   const bsa_tensor *out, const bsa_tensor *dout, const bsa_tensor *lse,
                   const bsa_tensor *index, const bsa_tensor *cu_seqlens_q,
                   const bsa_tensor *cu_seqlens_kv, const bsa_tensor *seqused_kv,
                   const bsa_tensor *block_table, const bsa_params *params,
                   const bsa_tensor *dq, const bsa_tensor *dk, const bsa_tensor *dv,
                   void *workspace, size_t workspace_bytes, void *stream);

/* ----------------------------------------------------- status, layout */
/* Synchronises `stream`, then copies the workspace's status word (the
 * BSA_FLAG_* bits raised by the last call that used this workspace). */
bsa_status bsa_read_status(const void *workspace, void *stream, uint32_t *flags);

const char *bsa_status_string(bsa_status status);

/* Where the builders' results sit inside a workspace, so that callers (and
 * the tests) can inspect them after a call.  Offsets are bytes from the
 * workspace start; unused regions have bytes == 0.
 *   status     uint32[16]: [0] flags, [2] forward items, [3] backward items
 *              claimed so far past the first one per CTA, [4] backward items,
 *              [5] total kv blocks TK, [6] inverse-index entries, [8..9] the
 *              inverse lists' 128-row query slices (uint64)
 *   batch      per batch 12 x int32: qlen, kvlen, nq, nk, qoff, koff,
 *              q_tok0 (2 words, int64), kv_tok0 (2 words, int64), kvst (kv
 *              rows stored for the batch), 1 spare
 *   comp       uint16 [Hidx][Rg][W] compacted index rows (0xFFFF padded)
 *   ncomp      int32 [Hidx][Rg] accepted entries per row
 *   fwd_items  int32 forward item ids in execution order
 *   inv_off    int32 [Hidx*TK+1] CSR offsets of the KV-major inverse
 *   inv_list   int32 batch-local query blocks per (index head, kv block)
 *   bwd_items  int32 backward item ids in the order the CTAs claim them:
 *              the items above 1/512 of the total cost first, longest
 *              first, then kv head by kv head, longest first within a head
 * Item ids: forward (h1*Rg + gq)*(BQ/128) + q_slice, gq the global query
 * block row, each item 128 query rows of head h1; but when the index is
 * shared by the heads of a GQA group (Hidx == N2) with g = N1/N2 in
 * {2, 4, 8, 16}, the forward packs the group (GenericBlockSparseAttention
 * article, attribute isPackedGQA): (h2*Rg + gq)*(BQ*g/128) + slice, each item
 * query rows [slice*128/g, (slice+1)*128/g) of the block for all g heads of
 * kv head h2, so that every K/V chunk is streamed once for the group (the
 * deterministic backward's q-major pass keeps one head per item); backward (h2*TK + gk)*(BKV/128) + kv_slice, gk the global kv
 * block (batch b's blocks after those of every earlier batch) and TK the
 * total kv blocks of this call (status word [5]). */
typedef struct bsa_ws_region {
  uint64_t offset;
  uint64_t bytes;
} bsa_ws_region;

typedef struct bsa_ws_layout {
  bsa_ws_region status, batch, comp, ncomp, fwd_items, inv_off, inv_list, bwd_items;
  bsa_ws_region dsum, dq_acc, sort_keys;
  int64_t Rg;      /* global query-block rows (TND: R; BNSD: B*ceil(Sq/BQ)) */
  int64_t tk_max;  /* upper bound on total kv blocks, from shapes */
  uint64_t total_bytes;
} bsa_ws_layout;

bsa_status bsa_fwd_workspace_layout(const bsa_tensor *q, const bsa_tensor *k, const bsa_tensor *v,
                                    const bsa_tensor *index, const bsa_tensor *cu_seqlens_q,
                                    const bsa_tensor *cu_seqlens_kv, const bsa_tensor *seqused_kv,
                                    const bsa_tensor *block_table, const bsa_params *params,
                                    const bsa_tensor *out, const bsa_tensor *lse,
                                    bsa_ws_layout *layout);

bsa_status bsa_bwd_workspace_layout(const bsa_tensor *q, const bsa_tensor *k, const bsa_tensor *v,
                                    const bsa_tensor *out, const bsa_tensor *dout,
                                    const bsa_tensor *lse, const bsa_tensor *index,
                                    const bsa_tensor *cu_seqlens_q,
                                    const bsa_tensor *cu_seqlens_kv,
                                    const bsa_tensor *seqused_kv, const bsa_tensor *block_table,
                                    const bsa_params *params, const bsa_tensor *dq,
                                    const bsa_tensor *dk, const bsa_tensor *dv,
                                    bsa_ws_layout *layout);

/* Profiling hook (the pages have no counterpart).  The next bsa_fwd or
 * bsa_bwd call made by this host thread records `before` and `after`
 * (cudaEvent_t handles created by the caller, passed as void*) on its stream
 * immediately before and after its main attention kernel (the deterministic
 * backward: its two main kernels, kv-major dK/dV and q-major dQ), so that
 * kernel's duration can be timed apart from the preparation kernels; the setting is
 * then cleared, whatever the call's outcome: a call that launches nothing
 * (failed validation, an empty problem) records nothing.  Both NULL clears a
 * pending pair; exactly one NULL returns BSA_ERR_NULLPTR.  bsa_fwd_static_
 * workspace passes the pair on to its bsa_fwd. */
bsa_status bsa_set_main_kernel_events(void *before, void *after);

/* Diagnostic (the pages have no counterpart).  For n floats x (device
 * memory), writes y_poly[i] = an FMA-pipe 2^x (range reduction plus a degree-3
 * minimax polynomial, relative error <= 7.5e-5 for -126 <= x < 128, +inf from
 * 128 up; a building block no shipped kernel calls) and y_mufu[i] = the hardware
 * ex2.approx of x, asynchronously on `stream`.  Caller-owned device buffers;
 * BSA_ERR_NULLPTR for a NULL buffer with n > 0, BSA_ERR_PARAM_INVALID for
 * n < 0, BSA_ERR_CUDA if the launch fails. */
bsa_status bsa_selftest_exp2(const float *x, float *y_poly, float *y_mufu, int64_t n, void *stream);

/* Diagnostic (the pages have no counterpart).  Packs x[4i .. 4i+3] into
 * packed[i] as four E4M3 bytes (element 4i in the lowest byte; round to
 * nearest even, saturating to +-448), with the same routine the FP8 forward
 * uses for P.  n % 4 == 0; device pointers; asynchronous on `stream`. */
bsa_status bsa_selftest_e4m3(const float *x, uint32_t *packed, int64_t n, void *stream);

/* Diagnostic (the pages have no counterpart).  For n (even) float triples
 * a[i], b[i], c[i] (device memory) writes, with the paired fp32 instructions
 * of sm_100 (fma/add/mul .rn.f32x2, two elements per instruction) that the
 * backward kernels' softmax uses, pair[i] = fma(a,b,c), pair[n+i] = a+b,
 * pair[2n+i] = a*b, and the same three results from the scalar round-to-
 * nearest operations into scalar[0..3n): the two must agree bit for bit.
 * Caller-owned device buffers (pair and scalar 3n floats each); asynchronous
 * on `stream`; BSA_ERR_PARAM_INVALID for n < 0 or odd, BSA_ERR_NULLPTR for a
 * NULL buffer with n > 0, BSA_ERR_CUDA if the launch fails. */
bsa_status bsa_selftest_f32x2(const float *a, const float *b, const float *c, float *pair,
                              float *scalar, int64_t n, void *stream);

/* Diagnostic (the pages have no counterpart).  Launches one warp that waits
 * on a device barrier nothing ever completes, through the bounded wait every
 * kernel of this library uses: after its time limit (about 2 s) the wait
 * gives up, sets BSA_FLAG_TIMEOUT in flags[0] (a caller-owned device word,
 * zeroed by the caller) and the kernel returns, leaving the context usable.
 * Asynchronous on `stream`; BSA_ERR_NULLPTR for a NULL flags pointer. */
bsa_status bsa_selftest_wait_timeout(uint32_t *flags, void *stream);

/* Library ABI version (bumped on any signature or layout change; 2 added
 * bsa_params.mask_type, 3 bsa_params.deterministic). */
int32_t bsa_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* BSA_H_ */
