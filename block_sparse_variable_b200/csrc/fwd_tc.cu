// fwd_tc.cu -- tcgen05 / TMEM / TMA forward for sm_100a.
//
// Math (BlockSparseAttentionGrad README, "Formula"; BlitzSparseAttention,
// "softmax_lse output"): out = softmax(scale * Q K_sel^T) V_sel per query
// row over the kv tokens of the blocks in the row's compacted index row,
// lse = natural log of the sum of exp(scale * q.k).
//
// One persistent CTA per SM; each work item is 128 query rows of one head,
// walked over 128-row kv chunks t of the selected blocks.
// Warp roles (384 threads):
//   warp 8      TMA: the Q tile once per item, then K chunks (3-stage ring);
//               as an item's last index entry starts, the next item's Q tile
//               is prefetched into L2
//   warp 10     TMA: the matching V chunks (3-stage ring); every tile is one
//               5-D copy of both 64-column halves
//   warp 9      TMEM owner; issues O += P_t V_t (TS form, P read from TMEM)
//   warp 11     issues S_t = Q K_t^T (SS form), up to two chunks ahead of the
//               softmax.  The MMA issue is split over two schedulers because
//               an MMA issued into a full tensor-pipe queue stalls in issue and
//               holds up the softmax warps that share its scheduler.
//   warps 0..7  two softmax warpgroups; thread (group w, row r) owns kv
//               columns [64w, 64w+64) of query row r in every chunk.
//               P = exp2(s*scale*log2 e - m) is computed at once against the
//               current reference m (log2 domain); only when a half-row sum
//               of P exceeds 2^8 do the two warps on those rows exchange their
//               maxima, take a new m, recompute P and rescale O and the
//               partial sums l.  P overwrites the group's own S columns as
//               16-bit pairs.  Epilogue: out = O / (l_0 + l_1),
//               lse = (m + log2(l_0 + l_1)) ln 2.
// TMEM columns: three S/P buffers [0,128), [128,256), [256,384); O [384,384+D).
// Every mbarrier wait is bounded (2 s); on expiry the CTA raises
// BSA_FLAG_TIMEOUT, drains its in-flight copies and MMAs, frees TMEM and
// returns.  The two softmax warpgroups meet only on mbarriers, so an abort
// never strands one of them on a hardware barrier.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>

#include "addr.cuh"
#include "bsa_internal.h"
#include "fp8.cuh"
#include "fwd_walk.cuh"
#include "launch.cuh"
#include "pack16.cuh"
#include "sm100.cuh"
#include "tc_common.h"
#include "tc_device.cuh"

namespace bsa {
namespace {

using namespace sm100;

constexpr int kSoftmaxGroups = 2;  // warpgroups sharing the kv columns of a chunk
constexpr int kSoftmaxThreads = 128 * kSoftmaxGroups;
constexpr int kTcThreads = kSoftmaxThreads + 128;  // + Q/K loads, PV MMAs, V loads, S MMAs
constexpr int kStages = 3;       // depth of the K ring and of the V ring
constexpr int kSBufs = 3;        // S / P buffers in TMEM
constexpr int kLoadWarp = 4 * kSoftmaxGroups;
constexpr int kMmaWarp = kLoadWarp + 1;
constexpr int kVLoadWarp = kLoadWarp + 2;
constexpr int kSMmaWarp = kLoadWarp + 3;
constexpr int kCols = 128 / kSoftmaxGroups;  // kv columns per softmax thread
// a row takes a new reference max once its P could exceed 2^8 (a half-row
// sum of P above 2^8)
constexpr float kRescaleSum = 256.0f;

// barrier slots
enum : int {
  kBarQFull = 0,
  kBarQEmpty = 1,
  kBarKFull = 2,    // + K stage
  kBarKEmpty = 5,   // + K stage
  kBarVFull = 8,    // + V stage
  kBarVEmpty = 11,  // + V stage
  kBarSFull = 14,   // + S buffer
  kBarPFull = 17,   // + S buffer (one arrival per softmax thread)
  kBarPVDone = 20,  // + (chunk index & 1): P_t V_t is in O
  kBarXchg = 22,    // + row quarter: rendezvous of the warps that share 32 query
                    // rows (one per group; 32 arrivals per warp)
  kBarDrain = 26,   // the P V issuer's MMAs on the abort path
  kBarSFree = 27,   // + S buffer: the P V product that read the buffer's P is done
  kBarDrainS = 30,  // the S issuer's MMAs on the abort path
  kNumBars = 31
};

template <int D, bool kFp8>
struct Layout {
  static constexpr int kBox = 128 * 128;  // one 128-row x 128-byte box (64 16-bit / 128 8-bit columns)
  static constexpr int kTile = (kFp8 ? D / 128 : D / 64) * kBox;  // Q / K / V tile
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTile;
  static constexpr int kV = kK + kStages * kTile;
  static constexpr int kBars = kV + kStages * kTile;
  static constexpr int kFlags = kBars + kNumBars * 8;                 // [2][softmax warps] u32
  static constexpr int kXsum = kFlags + 2 * 4 * kSoftmaxGroups * 4;   // [2][groups][128] sums
  static constexpr int kTmemPtr = kXsum + 2 * kSoftmaxGroups * 128 * 4;
  static constexpr int kAbort = kTmemPtr + 4;
  static constexpr int kBytes = kAbort + 4;
  // the dynamic shared window starts 1024-byte aligned (checked at run time)
  static constexpr int kAlloc = kBytes;
  static_assert(kAlloc <= 232448, "shared memory budget");
};

template <bool kPack>
__device__ __forceinline__ ItemView item_of(const Problem &p, int id) {
  if constexpr (kPack) return item_view_packed(p, id);
  else return item_view(p, id);
}

// kFp8: q, k, v in e4m3 (kind::f8f6f4 MMAs; P cast to e4m3 before P V);
// BF16 then selects only the type of out.  kPack: packed-head items (the
// query heads of a GQA group share the index row; p.pack_g heads per tile).
template <int D, bool BF16, bool kCausal, bool kFp8, bool kPack>
__global__ void __launch_bounds__(kTcThreads, 1)
    k_fwd_tc(const Problem p, const __grid_constant__ CUtensorMap map_q,
             const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v) {
  static_assert(!kFp8 || D == 128, "FP8 tiles are one 128-byte box wide");
  using L = Layout<D, kFp8>;
  using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;  // out (and 16-bit inputs)
  extern __shared__ unsigned char smem_raw[];
  griddep_wait();
  griddep_launch_next();
  const uint32_t base = smem_u32(smem_raw);
  unsigned char *sbase = smem_raw;
  if (base & 1023u) {  // 128-byte swizzled tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) atomicOr(p.status + kStFlags, BSA_FLAG_INTERNAL);
    return;
  }
  const uint32_t sQ = base + L::kQ, sK = base + L::kK, sV = base + L::kV;
  auto bar = [&](int i) { return base + L::kBars + 8u * uint32_t(i); };
  volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(sbase + L::kTmemPtr);
  volatile int *abort = reinterpret_cast<volatile int *>(sbase + L::kAbort);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_items = int(p.status[kStFwdItems]);

  if (tid == 0) {
    mbar_init(bar(kBarQFull), 1);
    mbar_init(bar(kBarQEmpty), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
    }
    for (int b = 0; b < kSBufs; ++b) {
      mbar_init(bar(kBarSFull + b), 1);
      mbar_init(bar(kBarPFull + b), kSoftmaxThreads);
    }
    mbar_init(bar(kBarPVDone), 1);
    mbar_init(bar(kBarPVDone + 1), 1);
    for (int q = 0; q < 4; ++q) mbar_init(bar(kBarXchg + q), kSoftmaxThreads / 4);
    mbar_init(bar(kBarDrain), 1);
    mbar_init(bar(kBarDrainS), 1);
    for (int b = 0; b < kSBufs; ++b) mbar_init(bar(kBarSFree + b), 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(base + L::kTmemPtr, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS0 = tmem, tO = tmem + uint32_t(kSBufs) * 128u;

  if (warp == kLoadWarp || warp == kVLoadWarp) {
    // ----------------------------------------------------- TMA producers
    const bool is_k = warp == kLoadWarp;
    if (lane == 0) {
      const CUtensorMap *map = is_k ? &map_k : &map_v;
      if (is_k) tma_prefetch_desc(&map_q);
      tma_prefetch_desc(map);
      const uint32_t ring = is_k ? sK : sV;
      const int full0 = is_k ? kBarKFull : kBarVFull, empty0 = is_k ? kBarKEmpty : kBarVEmpty;
      uint32_t kv_it = 0, q_it = 0;
      int armed_q = -1, armed[kStages] = {-1, -1, -1};
      bool ok = true;
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        const ItemView v = item_of<kPack>(p, p.fwd_items[it]);
        if (settle(p, v, Chunk{0, 0}).x >= v.ncnt) continue;  // no chunk: nothing to load
        if (is_k) {
          if (!(ok = wait_bar_lazy(bar(kBarQEmpty), (q_it & 1u) ^ 1u, abort, p.status))) break;
          mbar_expect_tx(bar(kBarQFull), L::kTile);
          armed_q = int(q_it & 1u);
          const int tok = p.q_layout == BSA_LAYOUT_TND ? int(v.bi.q_tok0) + v.t0 : v.t0;
          const int bb = p.q_layout == BSA_LAYOUT_TND ? 0 : v.b;
          // packed heads: coordinates (0, row, first head, 0, batch)
          if constexpr (kPack) tma_load_5d(sQ, &map_q, bar(kBarQFull), 0, tok, v.h1, 0, bb);
          else tma_load_5d(sQ, &map_q, bar(kBarQFull), 0, tok, 0, v.h1, bb);
          ++q_it;
        }
        for (Chunk ch = settle(p, v, Chunk{0, 0}); ch.x < v.ncnt; ch = next_chunk(p, v, ch)) {
          const int s = int(kv_it % kStages);
          const uint32_t ph = (kv_it / kStages) & 1u;
          const int u0 = v.u0(ch);
          int pg;
          page_ok(p, v, u0, pg);
          int row, last;  // tile coordinates: (0, row, 0, h2, last)
          if (p.kv_layout == BSA_LAYOUT_PA_BBND) { row = u0 % p.page_size; last = pg; }
          else if (p.kv_layout == BSA_LAYOUT_TND) { row = int(v.bi.kv_tok0) + u0; last = 0; }
          else { row = u0; last = v.b; }
          if (!(ok = wait_bar_lazy(bar(empty0 + s), ph ^ 1u, abort, p.status))) break;
          mbar_expect_tx(bar(full0 + s), L::kTile);
          armed[s] = int(ph);
          tma_load_5d(ring + s * L::kTile, map, bar(full0 + s), 0, row, 0, v.h2, last);
          if (is_k && ch.x == v.ncnt - 1 && ch.c == 0 && it + int(gridDim.x) < n_items) {
            // the next item's Q tile into L2 as this item's last index entry
            // starts: its load waits for this item's last S, and a miss to
            // memory then would stall the pipeline
            const ItemView w = item_of<kPack>(p, p.fwd_items[it + gridDim.x]);
            const int wtok = p.q_layout == BSA_LAYOUT_TND ? int(w.bi.q_tok0) + w.t0 : w.t0;
            const int wb = p.q_layout == BSA_LAYOUT_TND ? 0 : w.b;
            if constexpr (kPack) tma_prefetch_l2_5d(&map_q, 0, wtok, w.h1, 0, wb);
            else tma_prefetch_l2_5d(&map_q, 0, wtok, 0, w.h1, wb);
          }
          ++kv_it;
        }
      }
      if (*abort) {  // let every copy already issued land before the CTA exits
        if (armed_q >= 0) drain_wait(bar(kBarQFull), uint32_t(armed_q));
        for (int s = 0; s < kStages; ++s)
          if (armed[s] >= 0) drain_wait(bar(full0 + s), uint32_t(armed[s]));
      }
    }
  } else if (warp == kMmaWarp || warp == kSMmaWarp) {
    // -------------------------------------------------------- MMA issuers
    // Two warps on two different schedulers issue the MMAs: an MMA issued
    // into a full tensor-pipe queue stalls in issue and holds up the softmax
    // warps that share its scheduler, so the load is split.  S_t = Q K_t^T
    // (SS form) and O += P_t V_t (TS form, P read from TMEM) are independent
    // chains; S_t overwrites the buffer of P_{t-3} only after P_{t-3} V_{t-3}
    // is done (S_free).  Each warp runs its loop warp-uniformly (descriptors
    // precomputed and advanced by adding to their address field) and one
    // elected lane issues each MMA and commit.
    // (format 0 is E4M3 under kind::f8f6f4)
    constexpr uint32_t idS = idesc_f16(kFp8 ? false : BF16, 128, 128, false, false);
    constexpr uint32_t idPV = idesc_f16(kFp8 ? false : BF16, 128, D, false, true);
    // descriptors: K-major Q / K (a K step, 16 16-bit or 32 8-bit elements, is
    // +32 B; the second 64-column 16-bit box +16 KB); MN-major V (a K step is
    // 16 rows = +2 KB, or 32 rows = +4 KB for 8-bit; the two 64-column 16-bit
    // halves 16 KB apart)
    constexpr int kSSteps = kFp8 ? D / 32 : D / 16;
    constexpr int kPVSteps = kFp8 ? 4 : 8;
    const uint64_t dQ = sw128_desc(sQ, 16, 1024);
    const uint64_t dK = sw128_desc(sK, 16, 1024);
    const uint64_t dV = sw128_desc(sV, L::kBox, 1024);
    auto kstep = [](int kk) { return uint64_t((kk >> 2) * (L::kBox >> 4) + (kk & 3) * 2); };
    // 16 16-bit (or 32 8-bit) kv columns of P = 8 TMEM columns; the first 64
    // kv columns' P is in TMEM columns [0, 32) ([0, 16) for 8-bit), the next
    // 64's in [64, 96) ([64, 80)) of the S buffer
    auto pcol = [](int kk) {
      return kFp8 ? uint32_t(64 * (kk >> 1) + 8 * (kk & 1)) : uint32_t(64 * (kk >> 2) + 8 * (kk & 3));
    };
    const bool is_s = warp == kSMmaWarp;
    uint32_t kv_it = 0, q_it = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
      const ItemView v = item_of<kPack>(p, p.fwd_items[it]);
      const int n = count_chunks_warp(p, v, lane);
      if (n == 0) continue;
      if (is_s) {
        if (!(ok = wait_warp(bar(kBarQFull), q_it & 1u, abort, p.status))) break;
        ++q_it;
        for (int j = 0; j < n && ok; ++j) {
          const uint32_t t = kv_it + uint32_t(j);
          const int b = int(t % kSBufs), st = int(t % kStages);
          if (t >= uint32_t(kSBufs) &&
              !(ok = wait_warp(bar(kBarSFree + b), (t / kSBufs - 1) & 1u, abort, p.status)))
            break;
          if (!(ok = wait_warp(bar(kBarKFull + st), (t / kStages) & 1u, abort, p.status))) break;
          tc_fence_after();
          const uint32_t da = tS0 + uint32_t(b) * 128u;
          const uint64_t ka = dK + uint64_t(st * (L::kTile >> 4));
#pragma unroll
          for (int kk = 0; kk < kSSteps; ++kk) {
            if constexpr (kFp8) mma_ss_f8_e(da, dQ + kstep(kk), ka + kstep(kk), idS, kk > 0 ? 1u : 0u);
            else mma_ss_e(da, dQ + kstep(kk), ka + kstep(kk), idS, kk > 0 ? 1u : 0u);
          }
          mma_commit_e(bar(kBarSFull + b));
          mma_commit_e(bar(kBarKEmpty + st));
          if (j == n - 1) mma_commit_e(bar(kBarQEmpty));
        }
      } else {
        for (int j = 0; j < n && ok; ++j) {
          const uint32_t t = kv_it + uint32_t(j);
          const int b = int(t % kSBufs), st = int(t % kStages);
          if (!(ok = wait_warp(bar(kBarVFull + st), (t / kStages) & 1u, abort, p.status))) break;
          // P_t written (and, for a partial chunk, the V rows past the used
          // length zeroed by the softmax warps)
          if (!(ok = wait_warp(bar(kBarPFull + b), (t / kSBufs) & 1u, abort, p.status))) break;
          tc_fence_after();
          const uint32_t pa = tS0 + uint32_t(b) * 128u;
          const uint64_t vd = dV + uint64_t(st * (L::kTile >> 4));
#pragma unroll
          for (int kk = 0; kk < kPVSteps; ++kk)
            if constexpr (kFp8) mma_ts_f8_e(tO, pa + pcol(kk), vd + uint64_t(kk * 256), idPV, (j == 0 && kk == 0) ? 0u : 1u);
            else mma_ts_e(tO, pa + pcol(kk), vd + uint64_t(kk * 128), idPV, (j == 0 && kk == 0) ? 0u : 1u);
          mma_commit_e(bar(kBarPVDone + int(t & 1u)));
          mma_commit_e(bar(kBarVEmpty + st));
          mma_commit_e(bar(kBarSFree + b));
        }
      }
      kv_it += uint32_t(n);
    }
    if (*abort) {  // let issued MMAs finish before TMEM is freed
      const int dr = is_s ? kBarDrainS : kBarDrain;
      mma_commit_e(bar(dr));
      if (lane == 0) drain_wait(bar(dr), 0);
    }
    __syncwarp();
  } else if (warp < kLoadWarp) {
    // --------------------------------------------- softmax warpgroups
    const int wg = warp >> 2;
    const int r = tid & 127;  // tile row = TMEM lane
    // the query row and head of tile row r (packed heads: 128/g rows per head)
    const int rq = kPack ? r % (128 / p.pack_g) : r;
    const int rh = kPack ? r / (128 / p.pack_g) : 0;
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
    volatile uint32_t *flags = reinterpret_cast<volatile uint32_t *>(sbase + L::kFlags);
    float *xsum = reinterpret_cast<float *>(sbase + L::kXsum);
    const float kLn2 = 0.6931471805599453f;
    constexpr int kWarps = 4 * kSoftmaxGroups;
    uint32_t kv_it = 0, x_it = 0, item_n = 0;  // chunk counter; rendezvous counter; items done
    bool ok = true;
    // the warps holding the same 32 query rows (one per group) meet here
    // (bounded: an aborted peer cannot strand us)
    auto rendezvous = [&]() {
      mbar_arrive(bar(kBarXchg + (warp & 3)));
      ok = wait_warp(bar(kBarXchg + (warp & 3)), x_it & 1u, abort, p.status);
      ++x_it;
      return ok;
    };
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
      float m = -INFINITY, l = 0.f;
      int n = 0;
      {
        // the chunk walk needs only the index row, its length, kvlen and the
        // batch; the rest of the item is re-derived for the epilogue
        ItemView v;
        int coff;  // causal: the last kv token this row sees
        {
          const ItemView full = item_of<kPack>(p, p.fwd_items[it]);
          v.crow = full.crow;
          v.ncnt = full.ncnt;
          v.kvlen = full.kvlen;
          v.b = full.b;
          v.ksl = p.ksl;
          v.BKV = p.BKV;
          coff = kCausal ? full.t0 + rq + full.kvlen - full.bi.qlen : 0;
        }
        for (Cursor ck = cur_begin(p, v); ck.x < v.ncnt && ok; cur_next(p, v, ck), ++n, ++kv_it) {
          const int b = int(kv_it % kSBufs);
          if (!(ok = wait_warp(bar(kBarSFull + b), (kv_it / kSBufs) & 1u, abort, p.status))) break;
          tc_fence_after();
          const uint32_t tS = tS0 + uint32_t(b) * 128u + lane_off;
          const int u0c = cur_u0(v, ck);
          const int valid_all = v.kvlen - u0c;             // kv columns of the chunk that exist
          // the chunk columns this row may see (causal: up to its own token)
          const int vis_all = kCausal ? min(valid_all, coff - u0c + 1) : valid_all;
          const int valid = vis_all - kCols * wg;          // of this group's columns
          if (valid_all < 128) {
            // kv rows past the used length may hold anything (the rest of a
            // page, another sequence's tokens, even NaN); their P is (nearly)
            // 0, so make their V exactly 0 as well (before P is published:
            // the MMA reads V after P_full)
            const int st = int(kv_it % kStages);
            if (!(ok = wait_warp(bar(kBarVFull + st), (kv_it / kStages) & 1u, abort, p.status))) break;
            uint4 *vt = reinterpret_cast<uint4 *>(sbase + L::kV + st * L::kTile);
            const int per_half = (128 - valid_all) * 8;  // 16-byte words per 128-byte box
            for (int w = tid; w < per_half * (L::kTile / L::kBox); w += kSoftmaxThreads) {
              const int h = w / per_half, x = w % per_half;
              vt[h * (L::kBox / 16) + valid_all * 8 + x] = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
          }
          uint32_t x[kCols];
          tmem_ld_cols<kCols>(tS + uint32_t(kCols * wg), x);
          tmem_wait_ld();
          if (valid < kCols) {
#pragma unroll
            for (int c = 0; c < kCols; ++c)
              if (c >= valid) x[c] = __float_as_uint(-INFINITY);
          }
          // P = exp2(scale*log2(e)*s - m) over this group's columns, with the
          // row sum of this half
          float ps[2] = {0.f, 0.f};
          uint32_t pk[kCols / 2];
          auto exps = [&](float mm) {
            ps[0] = ps[1] = 0.f;
#pragma unroll
            for (int c = 0; c < kCols; c += 2) {
              const float a0 = fmaf(__uint_as_float(x[c]), p.scale_log2, -mm);
              const float a1 = fmaf(__uint_as_float(x[c + 1]), p.scale_log2, -mm);
              const float e0 = ex2(a0);
              const float e1 = ex2(a1);
              ps[(c >> 1) & 1] += e0 + e1;
              if constexpr (kFp8) {
                // P in e4m3, four to a 32-bit column (the pair before is in
                // pk[c >> 2]'s low half until this pair completes it)
                if ((c & 2) == 0) pk[c >> 2] = __float_as_uint(e0), pk[(c >> 2) + kCols / 4] = __float_as_uint(e1);
                else pk[c >> 2] = pack_e4m3x4(__uint_as_float(pk[c >> 2]), __uint_as_float(pk[(c >> 2) + kCols / 4]), e0, e1);
              } else {
                pk[c >> 1] = Pack2<T>::pack(e0, e1);
              }
            }
          };
          const bool first = m == -INFINITY;
          // After the first chunk P is computed at once against the current
          // reference m; the half-row max only decides whether the row needs
          // a new reference (rare), in which case P is computed again.
          if (!first) exps(m);
          auto half_max = [&]() {
            float pm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < kCols; ++c) pm[c & 3] = fmaxf(pm[c & 3], __uint_as_float(x[c]));
            return fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])) * p.scale_log2;
          };
          // does any row of this warp's columns need a new reference?  After
          // the first chunk the half-row sum of P decides: below 2^8 every P
          // is below 2^8 (a larger sum may call for a new reference that turns
          // out to change little, which is still exact); no max is needed.
          // (the first chunk of an item always takes a reference: both groups
          // know that without exchanging flags)
          // (a row whose visible scores are all still masked keeps m = -inf
          // and always asks for a reference)
          uint32_t any = 1;
          if (kCausal ? n > 0 : !first) {
            const uint32_t need =
                __any_sync(0xffffffffu, (kCausal && first) || !(ps[0] + ps[1] <= kRescaleSum)) ? 1u : 0u;
            if (lane == 0) flags[(kv_it & 1u) * kWarps + warp] = need;
            if (!rendezvous()) break;
            // one decision for the rows of this warp, shared with the other
            // group's warp on the same rows, so that both take the same path
            any = 0;
#pragma unroll
            for (int g2 = 0; g2 < kSoftmaxGroups; ++g2) any |= flags[(kv_it & 1u) * kWarps + 4 * g2 + (warp & 3)];
          }
          float alpha = 1.f;
          const bool grow = any != 0u;
          if (grow) {
            // the full row max: the other groups' columns are still S in TMEM
            float cm = half_max();
#pragma unroll 1
            for (int g2 = 0; g2 < kSoftmaxGroups; ++g2) {
              if (g2 == wg) continue;
              float ym = -INFINITY;
#pragma unroll 1
              for (int h = 0; h < 2; ++h) {  // in halves: fewer live registers
                uint32_t y[kCols / 2];
                tmem_ld_cols<kCols / 2>(tS + uint32_t(kCols * g2 + (kCols / 2) * h), y);
                tmem_wait_ld();
                const int vy = vis_all - kCols * g2 - (kCols / 2) * h;
#pragma unroll
                for (int c = 0; c < kCols / 2; ++c)
                  if (c < vy) ym = fmaxf(ym, __uint_as_float(y[c]));
              }
              cm = fmaxf(cm, ym * p.scale_log2);
            }
            // nobody overwrites S with P before every thread has read it
            if (!rendezvous()) break;
            const float m_new = fmaxf(m, cm);
            alpha = first ? 1.f : ex2(m - m_new);
            m = m_new;
            exps(!kCausal || m > -INFINITY ? m : 0.f);  // nothing visible yet: every P is 0
          }
          // P over the first half of this group's own S columns: no other
          // warp reads them any more (the grow path's reads of the other
          // group's S precede its rendezvous)
          tmem_st_cols<kFp8 ? kCols / 4 : kCols / 2>(tS + uint32_t(kCols * wg), pk);
          l = l * alpha + (ps[0] + ps[1]);
          if (grow && (kCausal || !first) && __any_sync(0xffffffffu, (!kCausal || !first) && alpha != 1.f)) {
            // O may only be rescaled once P_{t-1} V_{t-1} (and so every
            // earlier product, the tensor pipe being in order) has landed
            const uint32_t t = kv_it - 1;
            if (!(ok = wait_warp(bar(kBarPVDone + int(t & 1u)), (t / 2) & 1u, abort, p.status))) break;
            tc_fence_after();
            const uint32_t col = tO + lane_off + uint32_t(wg * (D / kSoftmaxGroups));
            uint32_t o[D / kSoftmaxGroups];
            tmem_ld_cols<D / kSoftmaxGroups>(col, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < D / kSoftmaxGroups; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st_cols<D / kSoftmaxGroups>(col, o);
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar(kBarPFull + b));
        }
      }
      if (!ok) break;
      // ---- epilogue: out = O / sum of the groups' l; group w writes D/4 columns
      const ItemView v = item_of<kPack>(p, p.fwd_items[it]);
      const bool live = rq < v.rows;
      T *orow = static_cast<T *>(p.out) + q_row(p.o_sb, p.o_sh, p.o_st, v.bi, v.b, v.h1 + rh, v.t0 + rq);
      if (n > 0) {
        const uint32_t t = kv_it - 1;  // the item's last P V; earlier ones precede it
        if (!(ok = wait_warp(bar(kBarPVDone + int(t & 1u)), (t / 2) & 1u, abort, p.status))) break;
        tc_fence_after();
      }
      constexpr int kOc = D / kSoftmaxGroups;  // output columns per group
      // the row sums of the groups, through slots alternating by item (the
      // partner reads this item's slot before it can write the slot again)
      float *xs = xsum + (item_n & 1u) * (kSoftmaxGroups * 128);
      xs[wg * 128 + r] = l;
      if (!rendezvous()) break;
      float Lsum = 0.f;
#pragma unroll
      for (int g2 = 0; g2 < kSoftmaxGroups; ++g2) Lsum += xs[g2 * 128 + r];
      if (wg == 0 && live && p.lse)
        p.lse[q_row(p.l_sb, p.l_sh, p.l_st, v.bi, v.b, v.h1 + rh, v.t0 + rq)] =
            Lsum > 0.f ? (m + __log2f(Lsum)) * kLn2 : -INFINITY;
      const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
      if (n > 0) {
        uint32_t o[kOc];
        tmem_ld_cols<kOc>(tO + lane_off + uint32_t(wg * kOc), o);
        tmem_wait_ld();
        if (live) {
#pragma unroll
          for (int c8 = 0; c8 < kOc / 8; ++c8) {
            uint4 w;
            w.x = Pack2<T>::pack(__uint_as_float(o[8 * c8]) * inv, __uint_as_float(o[8 * c8 + 1]) * inv);
            w.y = Pack2<T>::pack(__uint_as_float(o[8 * c8 + 2]) * inv, __uint_as_float(o[8 * c8 + 3]) * inv);
            w.z = Pack2<T>::pack(__uint_as_float(o[8 * c8 + 4]) * inv, __uint_as_float(o[8 * c8 + 5]) * inv);
            w.w = Pack2<T>::pack(__uint_as_float(o[8 * c8 + 6]) * inv, __uint_as_float(o[8 * c8 + 7]) * inv);
            reinterpret_cast<uint4 *>(orow + wg * kOc)[c8] = w;
          }
        }
      } else if (live) {
#pragma unroll
        for (int c = 0; c < kOc / 8; ++c)
          reinterpret_cast<uint4 *>(orow + wg * kOc)[c] = make_uint4(0, 0, 0, 0);
      }
      // O is free once every softmax thread has arrived on the next item's
      // first P_full (the P V issuer waits for it), so no rendezvous here
      tc_fence_before();
      ++item_n;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, bool BF16, bool kCausal, bool kFp8, bool kPack>
cudaError_t launch_tc2(const Problem &p, const FwdMaps &m, cudaStream_t s) {
  // at least 120 KB so that exactly one CTA (the sole owner of all 512 TMEM
  // columns) is resident per SM
  const int smem = Layout<D, kFp8>::kAlloc > 120 * 1024 ? Layout<D, kFp8>::kAlloc : 120 * 1024;
  cudaError_t e = cudaFuncSetAttribute(k_fwd_tc<D, BF16, kCausal, kFp8, kPack>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = p.fwd_slots < num_sms() ? p.fwd_slots : num_sms();
  if (grid <= 0) return cudaSuccess;
  e = launch_dep(k_fwd_tc<D, BF16, kCausal, kFp8, kPack>, dim3(unsigned(grid)), dim3(kTcThreads), size_t(smem), s,
                 p, m.q, m.k, m.v);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// packed-head items are a separate instantiation: the one-head kernel carries
// none of their row mapping
template <int D, bool BF16, bool kCausal, bool kFp8 = false>
cudaError_t launch_tc(const Problem &p, const FwdMaps &m, cudaStream_t s) {
  return p.pack_g > 1 ? launch_tc2<D, BF16, kCausal, kFp8, true>(p, m, s)
                      : launch_tc2<D, BF16, kCausal, kFp8, false>(p, m, s);
}

}  // namespace

cudaError_t launch_fwd_main(const Problem &p, cudaStream_t s) {
  FwdMaps m;
  cudaError_t e = make_fwd_maps(p, m);
  if (e != cudaSuccess) return e;
  // the causal mask and the e4m3 inputs are separate instantiations: the
  // plain kernel carries neither
  if (p.dtype == BSA_F8E4M3) {  // D = 128 (checked on the host); out_dtype picks the output type
    const bool ob = p.out_dtype == BSA_BF16;
    if (p.causal) return ob ? launch_tc<128, true, true, true>(p, m, s) : launch_tc<128, false, true, true>(p, m, s);
    return ob ? launch_tc<128, true, false, true>(p, m, s) : launch_tc<128, false, false, true>(p, m, s);
  }
  if (p.causal) {
    if (p.dtype == BSA_BF16)
      return p.D == 64 ? launch_tc<64, true, true>(p, m, s) : launch_tc<128, true, true>(p, m, s);
    return p.D == 64 ? launch_tc<64, false, true>(p, m, s) : launch_tc<128, false, true>(p, m, s);
  }
  if (p.dtype == BSA_BF16)
    return p.D == 64 ? launch_tc<64, true, false>(p, m, s) : launch_tc<128, true, false>(p, m, s);
  return p.D == 64 ? launch_tc<64, false, false>(p, m, s) : launch_tc<128, false, false>(p, m, s);
}

}  // namespace bsa
