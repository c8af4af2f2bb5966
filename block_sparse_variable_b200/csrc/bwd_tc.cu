// bwd_tc.cu -- tcgen05 / TMEM / TMA backward main kernel for sm_100a.
//
// BlockSparseAttentionGrad README, "Formula", in the stage order of the
// aclnnFlashAttentionUnpaddingScoreGradV2 article, section 8.3 (recompute p,
// dp, ds, dq, dk, dv).  KV-major: one work item is a 128-row kv chunk of kv
// head h2; its K and V stay in shared memory and dK, dV accumulate in TMEM
// while the item walks, for every q head of the GQA group, the query blocks
// that selected its kv block (the inverted index) in 128-row q steps:
//   phase 1:
//     S^T  = K Q^T          -> TMEM R0        (M = kv, N = q, K = D), issued
//                              as soon as the previous step's phase 2 is done
//     dP^T = V dOut^T       -> TMEM R1        once the previous dQ left R1
//   softmax warps (thread = kv row, group w = q columns [64w, 64w+64)):
//     P^T  = exp2(scale*log2(e)*S^T - lse*log2(e))   (0 for rows/cols outside)
//     dS^T = P^T o (dP^T - Dsum)
//     P and dS packed to 16-bit pairs into the group's own R0 columns (the
//     TS-form A operands) and dS also into shared memory (for dQ)
//   phase 2 (three interleaved MMA chains):
//     dV  += P^T dOut       (A from TMEM)
//     dK  += dS^T Q         (A from TMEM)
//     dQ_s = dS K           -> TMEM R1        (A = dS from shared memory)
//   the softmax warps then stage dQ_s (fp32) in shared memory over the
//   step's Q and dOut tiles and the TMA warp has the TMA unit add it into the
//   global dQ accumulator (bulk tensor reductions, which run on while the
//   next steps compute); after the item, dK * scale and dV are stored.
// TMEM columns: R0 [0,128), R1 [128,256), dV [256,256+D), dK [384,384+D).
// Items of a kv head that share a query list start their walks at different
// entries so that their dQ reductions do not meet on the same rows.
// Warp roles (320 threads): 0..7 the two groups, 8 TMA (K, V per item; Q,
// dOut per step into a 2-slot ring, with lse and Dsum staged by its lanes;
// the dQ reductions of the step that held a slot before), 9 TMEM owner and
// MMA issuer.  Every mbarrier wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <type_traits>

#include "addr.cuh"
#include "bsa_internal.h"
#include "f32x2.cuh"
#include "launch.cuh"
#include "pack16.cuh"
#include "sm100.cuh"
#include "tc_common.h"
#include "tc_device.cuh"

namespace bsa {
namespace {

using namespace sm100;

constexpr int kBThreads = 320;
constexpr int kBLoadWarp = 8;
constexpr int kBMmaWarp = 9;

enum : int {
  kBarKV = 0,       // K, V of the item landed
  kBarKVEmpty = 1,  // the item's MMAs are done with K, V
  kBarQD = 2,       // + slot: Q, dOut, lse, Dsum of a step landed
  kBarS = 4,        // S^T, dP^T of the step are in TMEM
  kBarDS = 5,       // P, dS written (256 arrivals)
  kBarP2 = 6,       // the step's dV, dK, dQ MMAs are done
  kBarDQOut = 7,    // + slot: the step's dQ left TMEM and sits, staged, in
                    // the slot's Q and dOut tiles (256 arrivals)
  kBarAcc = 9,      // the item's dK, dV are final
  kBarAccFree = 10, // dK, dV read out (256 arrivals)
  kBarDrain = 11,
  kBarItemFull = 12,   // + ring slot: an item id is in the slot
  kBarItemEmpty = 16,  // + ring slot: every consumer warp has read it (9 arrivals)
  kNumBars = 20
};

// Work items are claimed at run time: a CTA's first item is its index, each
// further one the next unclaimed entry of the list (a global counter), so
// that the CTAs stay together on the list however unequal its items are.
// The TMA warp claims them and passes the ids to the MMA issuer and the
// softmax warps through a ring in shared memory.
constexpr int kRing = 4;
constexpr int kItemReaders = 9;  // the MMA warp and the eight softmax warps

template <int D>
struct BLayout {
  static constexpr int kBox = 128 * 128;
  static constexpr int kTile = (D / 64) * kBox;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTile;
  static constexpr int kQ = kV + kTile;       // [2 slots]
  static constexpr int kDO = kQ + 2 * kTile;  // [2 slots]
  static constexpr int kDS = kDO + 2 * kTile; // dS: 128 kv rows x 128 q (two 64-q regions)
  static constexpr int kStat = kDS + 2 * kBox;  // [2 slots][lse2 128 | Dsum 128] floats
  static constexpr int kBars = kStat + 2 * 256 * 4;
  static constexpr int kTmemPtr = kBars + kNumBars * 8;
  static constexpr int kAbort = kTmemPtr + 4;
  static constexpr int kStepT0 = kAbort + 4;  // [2 slots] first query row of the step
  static constexpr int kItems = kStepT0 + 2 * 4;  // [kRing] claimed item ids (-1: none left)
  static constexpr int kBytes = kItems + kRing * 4;
  static_assert(kBytes <= 232448, "shared memory budget");
};

struct BItem {
  int b, h2, u0, kvlen, wb, pg, gk, steps_ok, rot;
  BatchInfo bi;
};

__device__ __forceinline__ BItem b_item(const Problem &p, int id, int TK) {
  BItem v;
  const int ks = id % p.ksl;
  v.gk = (id / p.ksl) % TK;
  v.h2 = id / (p.ksl * TK);
  v.b = p.kb_batch[v.gk];
  v.bi = p.batch[v.b];
  const int j = v.gk - v.bi.koff;
  v.u0 = j * p.BKV + ks * 128;
  v.kvlen = v.bi.kvlen;
  v.wb = min(128, v.bi.kvst - v.u0);
  v.pg = p.kv_layout == BSA_LAYOUT_PA_BBND ? kv_page(p, v.b, v.u0) : 0;
  v.steps_ok = v.pg >= 0;
  // Items of one kv head that share a query list would otherwise walk it in
  // the same order at the same time and pile their dQ reductions onto the
  // same addresses; each starts at its own place in the list instead.
  v.rot = v.gk * p.ksl + ks;
  return v;
}

struct BStep {
  int hh, e, st;  // q head within the group, inverted-list entry, 128-row step
};

__device__ __forceinline__ int64_t b_list(const Problem &p, const BItem &v, int hh, int TK) {
  const int h1 = v.h2 * p.g + hh;
  const int hi = p.Hidx == p.N1 ? h1 : v.h2;
  return int64_t(hi) * TK + v.gk;
}

// q block of entry e (in walking order) of the item's list for q head hh
__device__ __forceinline__ int b_qblock(const Problem &p, const BItem &v, int hh, int e, int TK) {
  const int64_t li = b_list(p, v, hh, TK);
  const int off = p.inv_off[li], len = p.inv_off[li + 1] - off;
  return p.inv_list[off + (e + v.rot) % len];
}

__device__ __forceinline__ BStep b_settle(const Problem &p, const BItem &v, BStep c, int TK) {
  while (c.hh < p.g) {
    const int64_t li = b_list(p, v, c.hh, TK);
    const int len = p.inv_off[li + 1] - p.inv_off[li];
    if (c.e < len) {
      const int i = p.inv_list[p.inv_off[li] + (c.e + v.rot) % len];
      if (c.st < p.nsub && i * p.BQ + c.st * 128 < v.bi.qlen) return c;
      ++c.e;
      c.st = 0;
      continue;
    }
    ++c.hh;
    c.e = 0;
    c.st = 0;
  }
  return c;
}

__device__ __forceinline__ BStep b_next(const Problem &p, const BItem &v, BStep c, int TK) {
  ++c.st;
  return b_settle(p, v, c, TK);
}

__device__ __forceinline__ int b_t0(const Problem &p, const BItem &v, const BStep &c, int TK) {
  return b_qblock(p, v, c.hh, c.e, TK) * p.BQ + c.st * 128;
}

// The number of steps of an item (the walk of b_settle / b_next), by a whole
// converged warp, once per item.  Without the dQ product (the deterministic
// backward) the MMA issuer and the softmax warps count an item's steps this
// way and take each step's first query row from the TMA warp (shared memory)
// instead of walking the inverted index between two steps, which measured
// faster there (and slower with the dQ product, whose kernel keeps the walk).
__device__ __forceinline__ int b_count_steps_warp(const Problem &p, const BItem &v, int TK, int lane) {
  int n = 0;
  for (int hh = 0; hh < p.g; ++hh) {
    const int64_t li = b_list(p, v, hh, TK);
    const int off = p.inv_off[li], len = p.inv_off[li + 1] - off;
    for (int e = lane; e < len; e += 32) {
      const int rem = v.bi.qlen - p.inv_list[off + e] * p.BQ;  // query rows from the block start
      n += rem > 0 ? min(p.nsub, (rem + 127) / 128) : 0;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
  return n;
}

template <int D, bool BF16, bool kCausal, bool kDQ>
__global__ void __launch_bounds__(kBThreads, 1)
    k_bwd_tc(const Problem p, const __grid_constant__ CUtensorMap map_q,
             const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
             const __grid_constant__ CUtensorMap map_do, const __grid_constant__ CUtensorMap map_dq) {
  using L = BLayout<D>;
  using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  extern __shared__ unsigned char smem_raw[];
  griddep_wait();
  griddep_launch_next();
  const uint32_t base = smem_u32(smem_raw);
  unsigned char *sbase = smem_raw;
  if (base & 1023u) {  // 128-byte swizzled tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) atomicOr(p.status + kStFlags, BSA_FLAG_INTERNAL);
    return;
  }
  const uint32_t sK = base + L::kK, sV = base + L::kV, sQ = base + L::kQ, sDO = base + L::kDO;
  const uint32_t sDS = base + L::kDS;
  float *stat = reinterpret_cast<float *>(sbase + L::kStat);
  int *step_t0 = reinterpret_cast<int *>(sbase + L::kStepT0);  // without dQ: per slot
  volatile int *items_ring = reinterpret_cast<volatile int *>(sbase + L::kItems);
  auto bar = [&](int i) { return base + L::kBars + 8u * uint32_t(i); };
  volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(sbase + L::kTmemPtr);
  volatile int *abort = reinterpret_cast<volatile int *>(sbase + L::kAbort);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_items = int(p.status[kStBwdItems]);
  const int TK = int(p.status[kStTK]);

  if (tid == 0) {
    mbar_init(bar(kBarKV), 1);
    mbar_init(bar(kBarKVEmpty), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarQD + s), 1);
      // with dQ: the softmax warps' 256 arrivals once the step's dQ is staged;
      // without: the MMA issuer's commit once the step's MMAs are done
      mbar_init(bar(kBarDQOut + s), kDQ ? 256 : 1);
    }
    mbar_init(bar(kBarS), 1);
    mbar_init(bar(kBarDS), 256);
    mbar_init(bar(kBarP2), 1);
    mbar_init(bar(kBarAcc), 1);
    mbar_init(bar(kBarAccFree), 256);
    mbar_init(bar(kBarDrain), 1);
    for (int r = 0; r < kRing; ++r) {
      mbar_init(bar(kBarItemFull + r), 1);
      mbar_init(bar(kBarItemEmpty + r), kItemReaders);
    }
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == kBMmaWarp) {
    tmem_alloc(base + L::kTmemPtr, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tR0 = tmem, tR1 = tmem + 128u, tdV = tmem + 256u, tdK = tmem + 384u;
  const float kLog2e = 1.4426950408889634f;

  // consumers: the next claimed item id from the ring (-1: none left, or abort)
  uint32_t cseq = 0;
  auto take_item = [&](bool &ok) -> int {
    const int r = int(cseq % kRing);
    if (!(ok = wait_warp(bar(kBarItemFull + r), (cseq / kRing) & 1u, abort, p.status))) return -1;
    const int it = items_ring[r];
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(kBarItemEmpty + r));
    ++cseq;
    return it;
  };

  if (warp == kBLoadWarp) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      tma_prefetch_desc(&map_do);
      tma_prefetch_desc(&map_dq);
    }
    uint32_t kv_it = 0, sk = 0;
    int armed_kv = -1, armed_qd[2] = {-1, -1};
    int pend_row[2] = {0, 0}, pend_h[2] = {0, 0};  // dQ origin of the step held in each slot
    bool ok = true;
    // A step is done with its slot once its dQ, staged there by the softmax
    // warps, has been handed to the TMA unit and read back out of shared
    // memory; the additions into global memory then proceed on their own.
    // One commit group per tile: the Q tile's boxes, then the dOut tile's.
    auto reduce_slot = [&](int sl) {
      if constexpr (kDQ) {
#pragma unroll
        for (int j = 0; j < D / 32; ++j) {
          const uint32_t src = j < D / 64 ? sQ + sl * L::kTile + j * L::kBox
                                          : sDO + sl * L::kTile + (j - D / 64) * L::kBox;
          tma_reduce_add_3d(&map_dq, src, 32 * j, pend_h[sl], pend_row[sl]);
          if (j == D / 64 - 1 || j == D / 32 - 1) bulk_commit();
        }
      }
    };
    auto flush = [&](uint32_t s) -> bool {  // the last two steps, after the loop
      const int sl = int(s & 1u);
      if (!wait_warp_lazy(bar(kBarDQOut + sl), (s >> 1) & 1u, abort, p.status)) return false;
      if (lane == 0) reduce_slot(sl);
      __syncwarp();
      return true;
    };
    // claim an item and hand its id (or -1 once the list is exhausted) to the
    // consumers
    uint32_t pseq = 0;
    auto publish = [&](int it) -> int {
      const int r = int(pseq % kRing);
      if (pseq >= uint32_t(kRing) &&
          !(ok = wait_warp_lazy(bar(kBarItemEmpty + r), (pseq / kRing - 1) & 1u, abort, p.status)))
        return -1;
      if (lane == 0) {
        items_ring[r] = it;
        mbar_arrive(bar(kBarItemFull + r));
      }
      __syncwarp();
      ++pseq;
      return it;
    };
    auto claim = [&]() -> int {
      int nx = 0;
      if (lane == 0) nx = int(gridDim.x) + int(atomicAdd(p.status + kStBwdNext, 1u));
      nx = __shfl_sync(0xffffffffu, nx, 0);
      return publish(nx < n_items ? nx : -1);
    };
    for (int it = publish(int(blockIdx.x) < n_items ? int(blockIdx.x) : -1); it >= 0 && ok; it = claim()) {
      const BItem v = b_item(p, p.bwd_items[it], TK);
      if (!v.steps_ok) continue;
      if (!(ok = wait_warp_lazy(bar(kBarKVEmpty), (kv_it & 1u) ^ 1u, abort, p.status))) break;
      if (lane == 0) {
        mbar_expect_tx(bar(kBarKV), 2 * L::kTile);
        armed_kv = int(kv_it & 1u);
        int row, last;  // tile coordinates: (0, row, 0, h2, last)
        if (p.kv_layout == BSA_LAYOUT_PA_BBND) { row = v.u0 % p.page_size; last = v.pg; }
        else if (p.kv_layout == BSA_LAYOUT_TND) { row = int(v.bi.kv_tok0) + v.u0; last = 0; }
        else { row = v.u0; last = v.b; }
        tma_load_5d(sK, &map_k, bar(kBarKV), 0, row, 0, v.h2, last);
        tma_load_5d(sV, &map_v, bar(kBarKV), 0, row, 0, v.h2, last);
      }
      ++kv_it;
      // A step's inputs: its q head and first query row (the walk of the
      // inverted index) and the raw lse / Dsum of its 128 query rows (rows
      // past qlen: lse -inf, Dsum 0).  They are fetched one step ahead: with
      // the dQ product, while the TMA unit reads the previous dQ out of the
      // slot, so that the walk's dependent loads are not on the slot's path.
      auto fetch = [&](const BStep &c, int &h1, int &t0, float (&l2r)[4], float (&dsr)[4]) {
        h1 = v.h2 * p.g + c.hh;
        t0 = b_t0(p, v, c, TK);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int t = t0 + lane + 32 * i;
          l2r[i] = -INFINITY;
          dsr[i] = 0.f;
          if (t < v.bi.qlen) {
            l2r[i] = p.lse[q_row(p.l_sb, p.l_sh, p.l_st, v.bi, v.b, h1, t)];
            const int64_t srow = p.q_layout == BSA_LAYOUT_BNSD ? int64_t(v.b) * p.Sq + t : v.bi.q_tok0 + t;
            dsr[i] = p.dsum[srow * p.N1 + h1];
          }
        }
      };
      BStep c = b_settle(p, v, BStep{0, 0, 0}, TK);
      int h1 = 0, t0 = 0;
      float l2r[4], dsr[4];
      if (c.hh < p.g) fetch(c, h1, t0, l2r, dsr);
      while (c.hh < p.g && ok) {
        const int slot = int(sk & 1u);
        // the step that held the slot before: its dQ is staged over the
        // slot's tiles; hand it to the TMA unit in two commit groups (Q tile,
        // dOut tile) so that each tile is refilled as soon as it is read out
        const bool refill = sk >= 2;
        if (refill && !(ok = wait_warp_lazy(bar(kBarDQOut + slot), ((sk - 2) >> 1) & 1u, abort, p.status))) break;
        // lse in log2 units, +inf for rows past qlen or with no selected key
        // (so P = 0), and Dsum; both staged negated, as the addends of the
        // softmax warps' paired fp32 operations
        float *st = stat + slot * 256;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float l2 = l2r[i] * kLog2e;
          st[lane + 32 * i] = -(l2 > -INFINITY ? l2 : INFINITY);
          st[128 + lane + 32 * i] = -dsr[i];
        }
        if constexpr (!kDQ)
          if (lane == 0) step_t0[slot] = t0;
        __syncwarp();
        const int tok = p.q_layout == BSA_LAYOUT_TND ? int(v.bi.q_tok0) + t0 : t0;
        const int bb = p.q_layout == BSA_LAYOUT_TND ? 0 : v.b;
        if (lane == 0) {
          if (kDQ && refill) reduce_slot(slot);
          mbar_expect_tx(bar(kBarQD + slot), 2 * L::kTile);
          armed_qd[slot] = int((sk >> 1) & 1u);
        }
        __syncwarp();
        const bool ahead = kDQ && refill;  // fetch while the slot is read out
        const BStep cn = b_next(p, v, c, TK);
        int h1n = 0, t0n = 0;
        float l2n[4] = {0.f, 0.f, 0.f, 0.f}, dsn[4] = {0.f, 0.f, 0.f, 0.f};
        if (ahead && cn.hh < p.g) fetch(cn, h1n, t0n, l2n, dsn);
        if (lane == 0) {
          if (kDQ && refill) bulk_wait_read<1>();
          tma_load_5d(sQ + slot * L::kTile, &map_q, bar(kBarQD + slot), 0, tok, 0, h1, bb);
          if (kDQ && refill) bulk_wait_read<0>();
          tma_load_5d(sDO + slot * L::kTile, &map_do, bar(kBarQD + slot), 0, tok, 0, h1, bb);
        }
        __syncwarp();
        if (!ahead && cn.hh < p.g) fetch(cn, h1n, t0n, l2n, dsn);
        pend_h[slot] = h1;
        pend_row[slot] = int((p.q_layout == BSA_LAYOUT_BNSD ? int64_t(v.b) * p.Sq : v.bi.q_tok0) + t0);
        ++sk;
        c = cn;
        h1 = h1n;
        t0 = t0n;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          l2r[i] = l2n[i];
          dsr[i] = dsn[i];
        }
      }
    }
    if (kDQ)
      for (uint32_t s = sk >= 2 ? sk - 2 : 0; s < sk && ok; ++s) ok = flush(s);
    if (*abort && lane == 0) {  // let every copy already issued land before the CTA exits
      if (armed_kv >= 0) drain_wait(bar(kBarKV), uint32_t(armed_kv));
      for (int s = 0; s < 2; ++s)
        if (armed_qd[s] >= 0) drain_wait(bar(kBarQD + s), uint32_t(armed_qd[s]));
    }
    if (kDQ && lane == 0) bulk_wait_all();  // every dQ addition has been made
  } else if (warp == kBMmaWarp) {
    // ------------------------------------------------------- MMA issuer
    constexpr uint32_t idSP = idesc_f16(BF16, 128, 128, false, false);  // S^T, dP^T
    constexpr uint32_t idKV = idesc_f16(BF16, 128, D, false, true);     // dV, dK
    constexpr uint32_t idQ = idesc_f16(BF16, 128, D, true, true);       // dQ
    const uint64_t dKk = sw128_desc(sK, 16, 1024), dVk = sw128_desc(sV, 16, 1024);
    const uint64_t dKmn = sw128_desc(sK, L::kBox, 1024);
    const uint64_t dDS = sw128_desc(sDS, L::kBox, 1024);
    auto kstep = [](int kk) { return uint64_t((kk >> 2) * (L::kBox >> 4) + (kk & 3) * 2); };
    uint32_t kv_it = 0, sk = 0, item_n = 0;
    bool ok = true;
    for (int it = take_item(ok); it >= 0 && ok; it = take_item(ok)) {
      const BItem v = b_item(p, p.bwd_items[it], TK);
      if (!v.steps_ok) continue;
      const int n_steps = kDQ ? 0 : b_count_steps_warp(p, v, TK, lane);
      // the previous item's dK, dV must have been read out
      if (item_n > 0 && !(ok = wait_warp(bar(kBarAccFree), (item_n - 1) & 1u, abort, p.status))) break;
      ++item_n;
      if (!(ok = wait_warp(bar(kBarKV), kv_it & 1u, abort, p.status))) break;
      ++kv_it;
      const int valid = v.kvlen - v.u0;
      if (valid < 128) {
        // kv rows past the used length (the rest of a page, another
        // sequence's tokens, padding) may hold anything, even NaN: zero them
        // in K and V so that they contribute nothing (valid >= 1: an item
        // exists only for a slice that starts below kvlen)
        for (int w = lane; w < (128 - valid) * 8 * (D / 64); w += 32) {
          const int h = w / ((128 - valid) * 8), x = w % ((128 - valid) * 8);
          reinterpret_cast<uint4 *>(sbase + L::kK + h * L::kBox)[valid * 8 + x] = make_uint4(0, 0, 0, 0);
          reinterpret_cast<uint4 *>(sbase + L::kV + h * L::kBox)[valid * 8 + x] = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      bool first = true;
      int s = 0;  // steps taken (without dQ: against the item's step count)
      for (BStep c = kDQ ? b_settle(p, v, BStep{0, 0, 0}, TK) : BStep{0, 0, 0};
           (kDQ ? c.hh < p.g : s < n_steps) && ok; c = kDQ ? b_next(p, v, c, TK) : c, ++s) {
        const int slot = int(sk & 1u);
        if (!(ok = wait_warp(bar(kBarQD + slot), (sk >> 1) & 1u, abort, p.status))) break;
        // R0 held the previous step's P and dS until its phase-2 MMAs were
        // done: S^T may start while the previous dQ is still being read out
        if (sk > 0 && !(ok = wait_warp(bar(kBarP2), (sk - 1) & 1u, abort, p.status))) break;
        tc_fence_after();
        const uint64_t dQk = sw128_desc(sQ + slot * L::kTile, 16, 1024);
        const uint64_t dOk = sw128_desc(sDO + slot * L::kTile, 16, 1024);
        if (lane == 0) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tR0, dKk + kstep(kk), dQk + kstep(kk), idSP, kk > 0 ? 1u : 0u);
        }
        __syncwarp();
        // R1 still holds the previous step's dQ until it has been read out
        // (without dQ it held dP^T, read before the previous step's dS_full)
        if (kDQ && sk > 0 &&
            !(ok = wait_warp(bar(kBarDQOut + ((sk - 1) & 1u)), ((sk - 1) >> 1) & 1u, abort, p.status)))
          break;
        tc_fence_after();
        if (lane == 0) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tR1, dVk + kstep(kk), dOk + kstep(kk), idSP, kk > 0 ? 1u : 0u);
          mma_commit(bar(kBarS));
        }
        __syncwarp();
        if (!(ok = wait_warp(bar(kBarDS), sk & 1u, abort, p.status))) break;
        tc_fence_after();
        const uint64_t dQmn = sw128_desc(sQ + slot * L::kTile, L::kBox, 1024);
        const uint64_t dOmn = sw128_desc(sDO + slot * L::kTile, L::kBox, 1024);
        if (lane == 0) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t pcol = uint32_t(64 * (kk >> 2) + 8 * (kk & 3));
            const uint32_t acc = (first && kk == 0) ? 0u : 1u;
            mma_ts(tdV, tR0 + pcol, dOmn + uint64_t(kk * 128), idKV, acc);
            mma_ts(tdK, tR0 + 32u + pcol, dQmn + uint64_t(kk * 128), idKV, acc);
            if constexpr (kDQ) mma_ss(tR1, dDS + uint64_t(kk * 128), dKmn + uint64_t(kk * 128), idQ, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(kBarP2));
          if constexpr (!kDQ) mma_commit(bar(kBarDQOut + slot));  // the slot's Q, dOut are free
        }
        __syncwarp();
        first = false;
        ++sk;
      }
      if (!ok) break;
      if (lane == 0) {
        mma_commit(bar(kBarKVEmpty));
        mma_commit(bar(kBarAcc));
      }
      __syncwarp();
    }
    if (*abort && lane == 0) {  // let issued MMAs finish before TMEM is freed
      mma_commit(bar(kBarDrain));
      drain_wait(bar(kBarDrain), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------- the two softmax groups
    const int wg = warp >> 2;
    const int r = tid & 127;  // kv row (TMEM lane) of the softmax and the epilogue
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
    uint32_t sk = 0, item_n = 0;
    bool ok = true;
    for (int it = take_item(ok); it >= 0 && ok; it = take_item(ok)) {
      const BItem v = b_item(p, p.bwd_items[it], TK);
      if (!v.steps_ok) {
        if (tid == 0) atomicOr(p.status + kStFlags, BSA_FLAG_BAD_PAGE);
        continue;
      }
      const bool kv_ok = v.u0 + r < v.kvlen;
      int nsteps = 0;
      const int n_steps = kDQ ? 0 : b_count_steps_warp(p, v, TK, lane);
      for (BStep c = kDQ ? b_settle(p, v, BStep{0, 0, 0}, TK) : BStep{0, 0, 0};
           (kDQ ? c.hh < p.g : nsteps < n_steps) && ok; c = kDQ ? b_next(p, v, c, TK) : c) {
        const int slot = int(sk & 1u);
        int t0 = kDQ ? b_t0(p, v, c, TK) : 0;
        if (!(ok = wait_warp(bar(kBarQD + slot), (sk >> 1) & 1u, abort, p.status))) break;
        if constexpr (!kDQ) t0 = step_t0[slot];
        if (!(ok = wait_warp(bar(kBarS), sk & 1u, abort, p.status))) break;
        tc_fence_after();
        const float *lse2 = stat + slot * 256;
        const float *dsum = lse2 + 128;
        uint32_t pp[32], dd[32];
        // causal: column q (query row t0 + q) sees this kv row iff q >= qmin;
        // the masked variant runs only where a warp's columns cross the diagonal
        const int qmin = kCausal ? v.u0 + r - (v.kvlen - v.bi.qlen) - t0 : INT_MIN;
        auto softmax = [&](auto masked) {
          // 16-column blocks of S^T and dP^T, the next block's TMEM loads in
          // flight while this one is computed
          const uint32_t c0 = uint32_t(64 * wg);
          uint32_t xs[2][16], xd[2][16];
          tmem_ld16(tR0 + lane_off + c0, xs[0]);
          tmem_ld16(tR1 + lane_off + c0, xd[0]);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            if (k + 1 < 4) {
              tmem_ld16(tR0 + lane_off + c0 + uint32_t(16 * (k + 1)), xs[(k + 1) & 1]);
              tmem_ld16(tR1 + lane_off + c0 + uint32_t(16 * (k + 1)), xd[(k + 1) & 1]);
            }
            const uint32_t *bs = xs[k & 1], *bd = xd[k & 1];
#pragma unroll
            for (int c2 = 0; c2 < 16; c2 += 2) {
              const int q = int(c0) + 16 * k + c2;
              // lse2 and dsum hold -lse*log2(e) and -Dsum (pairs of columns)
              const float2 a2 = fma2(make_float2(__uint_as_float(bs[c2]), __uint_as_float(bs[c2 + 1])),
                                     make_float2(p.scale_log2, p.scale_log2),
                                     *reinterpret_cast<const float2 *>(lse2 + q));
              float p0 = kv_ok ? ex2(a2.x) : 0.f;
              float p1 = kv_ok ? ex2(a2.y) : 0.f;
              if constexpr (decltype(masked)::value) {
                p0 = q >= qmin ? p0 : 0.f;
                p1 = q + 1 >= qmin ? p1 : 0.f;
              }
              const float2 t2 = add2(make_float2(__uint_as_float(bd[c2]), __uint_as_float(bd[c2 + 1])),
                                     *reinterpret_cast<const float2 *>(dsum + q));
              const float2 s2 = mul2(make_float2(p0, p1), t2);
              const float s0 = s2.x, s1 = s2.y;
              pp[8 * k + (c2 >> 1)] = Pack2<T>::pack(p0, p1);
              dd[8 * k + (c2 >> 1)] = Pack2<T>::pack(s0, s1);
            }
            if (k + 1 < 4) tmem_wait_ld();
          }
        };
        if constexpr (kCausal) {
          if (__any_sync(0xffffffffu, qmin > 64 * wg))
            softmax(std::true_type{});
          else
            softmax(std::false_type{});
        } else {
          softmax(std::false_type{});
        }
        // P and dS into this group's own R0 columns (no other group reads
        // them as S), dS also into shared memory for the dQ product
        tmem_st32(tR0 + lane_off + uint32_t(64 * wg), pp);
        tmem_st32(tR0 + lane_off + uint32_t(64 * wg + 32), dd);
        if constexpr (kDQ) {
          // dS^T row r, q columns [64w, 64w+64): one 128-byte swizzled row
          uint4 *row = reinterpret_cast<uint4 *>(sbase + L::kDS + wg * L::kBox + r * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            row[c ^ (r & 7)] = make_uint4(dd[4 * c], dd[4 * c + 1], dd[4 * c + 2], dd[4 * c + 3]);
        }
        tmem_wait_st();
        if constexpr (kDQ) fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(kBarDS));
        if constexpr (!kDQ) {  // dQ comes from the q-major pass
          ++sk;
          ++nsteps;
          continue;
        }
        // dQ of the step (TMEM lanes = q rows) out to shared memory, where the
        // step's Q and dOut tiles were (free once its MMAs are done): four
        // boxes of 32 fp32 columns x 128 rows in the 128-byte swizzle, group
        // 0's in the Q tile and group 1's in the dOut tile.  The TMA warp adds
        // them into the global accumulator.  Rows past qlen are staged as
        // zeros: adding them changes nothing.
        if (!(ok = wait_warp(bar(kBarP2), sk & 1u, abort, p.status))) break;
        tc_fence_after();
        {
          const bool q_ok = t0 + r < v.bi.qlen;
          unsigned char *boxes = sbase + (wg == 0 ? L::kQ : L::kDO) + slot * L::kTile;
#pragma unroll
          for (int h = 0; h < D / 64; ++h) {
            uint32_t x[32];
            tmem_ld32(tR1 + lane_off + uint32_t((D / 2) * wg + 32 * h), x);
            tmem_wait_ld();
            uint4 *row = reinterpret_cast<uint4 *>(boxes + h * L::kBox + r * 128);
#pragma unroll
            for (int c = 0; c < 8; ++c)
              row[c ^ (r & 7)] = q_ok ? make_uint4(x[4 * c], x[4 * c + 1], x[4 * c + 2], x[4 * c + 3])
                                      : make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(kBarDQOut + slot));
        ++sk;
        ++nsteps;
      }
      if (!ok) break;
      // ---- epilogue: dK * scale and dV, group w writes columns [w*D/2, (w+1)*D/2)
      if (!(ok = wait_warp(bar(kBarAcc), item_n & 1u, abort, p.status))) break;
      tc_fence_after();
      if (r < v.wb) {
        T *dkr = static_cast<T *>(p.dk) + kv_row(p, p.dk_sb, p.dk_sh, p.dk_st, v.bi, v.b, v.h2, v.u0 + r, v.pg);
        T *dvr = static_cast<T *>(p.dv) + kv_row(p, p.dv_sb, p.dv_sh, p.dv_st, v.bi, v.b, v.h2, v.u0 + r, v.pg);
        if (nsteps == 0) {
#pragma unroll
          for (int c = 0; c < D / 16; ++c) {
            reinterpret_cast<uint4 *>(dkr + (D / 2) * wg)[c] = make_uint4(0, 0, 0, 0);
            reinterpret_cast<uint4 *>(dvr + (D / 2) * wg)[c] = make_uint4(0, 0, 0, 0);
          }
        }
      }
      if (nsteps > 0) {
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          const uint32_t col = uint32_t((D / 2) * wg + 32 * h);
          uint32_t xk[32], xv[32];
          tmem_ld32(tdK + lane_off + col, xk);
          tmem_ld32(tdV + lane_off + col, xv);
          tmem_wait_ld();
          if (r < v.wb) {
            T *dkr = static_cast<T *>(p.dk) + kv_row(p, p.dk_sb, p.dk_sh, p.dk_st, v.bi, v.b, v.h2, v.u0 + r, v.pg) + col;
            T *dvr = static_cast<T *>(p.dv) + kv_row(p, p.dv_sb, p.dv_sh, p.dv_st, v.bi, v.b, v.h2, v.u0 + r, v.pg) + col;
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
              uint4 wk, wv;
              wk.x = Pack2<T>::pack(__uint_as_float(xk[c]) * p.scale, __uint_as_float(xk[c + 1]) * p.scale);
              wk.y = Pack2<T>::pack(__uint_as_float(xk[c + 2]) * p.scale, __uint_as_float(xk[c + 3]) * p.scale);
              wk.z = Pack2<T>::pack(__uint_as_float(xk[c + 4]) * p.scale, __uint_as_float(xk[c + 5]) * p.scale);
              wk.w = Pack2<T>::pack(__uint_as_float(xk[c + 6]) * p.scale, __uint_as_float(xk[c + 7]) * p.scale);
              wv.x = Pack2<T>::pack(__uint_as_float(xv[c]), __uint_as_float(xv[c + 1]));
              wv.y = Pack2<T>::pack(__uint_as_float(xv[c + 2]), __uint_as_float(xv[c + 3]));
              wv.z = Pack2<T>::pack(__uint_as_float(xv[c + 4]), __uint_as_float(xv[c + 5]));
              wv.w = Pack2<T>::pack(__uint_as_float(xv[c + 6]), __uint_as_float(xv[c + 7]));
              *reinterpret_cast<uint4 *>(dkr + c) = wk;
              *reinterpret_cast<uint4 *>(dvr + c) = wv;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(kBarAccFree));
      ++item_n;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kBMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, bool BF16, bool kCausal, bool kDQ>
cudaError_t launch_bwd_tc(const Problem &p, const BwdMaps &m, cudaStream_t s) {
  const int smem = BLayout<D>::kBytes > 120 * 1024 ? BLayout<D>::kBytes : 120 * 1024;
  cudaError_t e = cudaFuncSetAttribute(k_bwd_tc<D, BF16, kCausal, kDQ>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = p.bwd_slots < num_sms() ? p.bwd_slots : num_sms();
  if (grid <= 0) return cudaSuccess;
  e = launch_dep(k_bwd_tc<D, BF16, kCausal, kDQ>, dim3(unsigned(grid)), dim3(kBThreads), size_t(smem), s,
                 p, m.q, m.k, m.v, m.dout, m.dq_acc);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// the causal mask and the deterministic mode (dQ left to the q-major pass)
// are separate instantiations: the plain kernel carries neither
template <bool kCausal, bool kDQ>
cudaError_t launch_bwd_for(const Problem &p, const BwdMaps &m, cudaStream_t s) {
  if (p.dtype == BSA_BF16)
    return p.D == 64 ? launch_bwd_tc<64, true, kCausal, kDQ>(p, m, s) : launch_bwd_tc<128, true, kCausal, kDQ>(p, m, s);
  return p.D == 64 ? launch_bwd_tc<64, false, kCausal, kDQ>(p, m, s) : launch_bwd_tc<128, false, kCausal, kDQ>(p, m, s);
}

}  // namespace

cudaError_t launch_bwd_main(const Problem &p, cudaStream_t s) {
  BwdMaps m;
  cudaError_t e = make_bwd_maps(p, m);
  if (e != cudaSuccess) return e;
  if (p.deterministic)
    return p.causal ? launch_bwd_for<true, false>(p, m, s) : launch_bwd_for<false, false>(p, m, s);
  return p.causal ? launch_bwd_for<true, true>(p, m, s) : launch_bwd_for<false, true>(p, m, s);
}

}  // namespace bsa
