// dq_tc.cu -- q-major dQ pass of the deterministic backward, tcgen05 / TMEM /
// TMA for sm_100a.
//
// BlockSparseAttentionGrad README, "Formula": dQ = scale * dS K with
// dS = P o (dP - Dsum), P = exp(scale * Q K^T - lse), dP = dOut V^T, over the
// selected kv tokens of each query row.  The kv-major backward kernel adds
// every step's dQ into an fp32 accumulator from many CTAs, in an order that
// varies from run to run; here each work item (the forward's: 128 query rows
// of one head) walks its own kv chunks in index order and keeps dQ in TMEM,
// so dq is bitwise the same on every run.  P and dS are recomputed from lse
// (no online softmax) and the result is written once, rounded to the dtype.
//
// Warp roles (384 threads):
//   warp 8      TMA: the item's Q and dOut tiles, then K chunks (2-stage ring);
//               as an item's last index entry starts, the next item's Q and
//               dOut tiles are prefetched into L2
//   warp 10     TMA: the matching V chunks (2-stage ring)
//   warp 11     issues S_t = Q K_t^T into S buffer t % 2 and dP_t = dOut V_t^T
//               into the dP buffer (SS form)
//   warp 9      TMEM owner; issues dQ += dS_t K_t (TS form: dS read from the
//               S buffer, K_t as the MN-major operand)
//   warps 0..7  two groups; thread (group w, row r) owns kv columns
//               [64w, 64w+64) of query row r: P = exp2(s*scale*log2 e -
//               lse*log2 e), dS = P (dP - Dsum), 16-bit pairs into the group's
//               own S columns; epilogue dq = dtype(scale * dQ).
// TMEM columns: S buffers [0,128), [128,256); dP [256,384); dQ [384,384+D).
// Every mbarrier wait is bounded (2 s); on expiry the CTA raises
// BSA_FLAG_TIMEOUT, drains its in-flight copies and MMAs, frees TMEM and
// returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <type_traits>

#include "addr.cuh"
#include "coalesce.cuh"
#include "bsa_internal.h"
#include "fwd_walk.cuh"
#include "f32x2.cuh"
#include "launch.cuh"
#include "pack16.cuh"
#include "sm100.cuh"
#include "tc_common.h"
#include "tc_device.cuh"

namespace bsa {
namespace {

using namespace sm100;

constexpr int kDGroups = 2;
constexpr int kDSoftmaxThreads = 128 * kDGroups;
constexpr int kDThreads = kDSoftmaxThreads + 128;
constexpr int kDStages = 2;  // K ring and V ring
constexpr int kDLoadWarp = 4 * kDGroups;
constexpr int kDQMmaWarp = kDLoadWarp + 1;
constexpr int kDVLoadWarp = kDLoadWarp + 2;
constexpr int kDSMmaWarp = kDLoadWarp + 3;

enum : int {
  kDBarQFull = 0,     // Q and dOut of the item landed
  kDBarQEmpty = 1,    // the item's S and dP MMAs are done with them
  kDBarKFull = 2,     // + stage
  kDBarKEmpty = 4,    // + stage: S_t and dQ_t are done with K_t
  kDBarVFull = 6,     // + stage
  kDBarVEmpty = 8,    // + stage: dP_t is done with V_t
  kDBarSFull = 10,    // + S buffer: S_t landed
  kDBarSFree = 12,    // + S buffer: dQ_t (which read dS_t there) is done
  kDBarDPFull = 14,   // dP_t landed
  kDBarDPFree = 15,   // dP_t read by every softmax thread (256 arrivals)
  kDBarDSFull = 16,   // + S buffer: dS_t written (256 arrivals)
  kDBarDQDone = 18,   // the item's last dQ MMA is done
  kDBarDrain = 19,    // the dQ issuer's MMAs on the abort path
  kDBarDrainS = 20,   // the S / dP issuer's MMAs on the abort path
  kDNumBars = 21
};

template <int D>
struct DLayout {
  static constexpr int kBox = 128 * 128;         // one 128-row x 64-col 16-bit box
  static constexpr int kTile = (D / 64) * kBox;
  static constexpr int kQ = 0;
  static constexpr int kDO = kQ + kTile;
  static constexpr int kK = kDO + kTile;
  static constexpr int kV = kK + kDStages * kTile;
  static constexpr int kBars = kV + kDStages * kTile;
  static constexpr int kTmemPtr = kBars + kDNumBars * 8;
  static constexpr int kAbort = kTmemPtr + 4;
  static constexpr int kBytes = kAbort + 4;
  static_assert(kBytes <= 232448, "shared memory budget");
};

template <int D, bool BF16, bool kCausal>
__global__ void __launch_bounds__(kDThreads, 1)
    k_dq_tc(const Problem p, const __grid_constant__ CUtensorMap map_q,
            const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
            const __grid_constant__ CUtensorMap map_do) {
  using L = DLayout<D>;
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
  const uint32_t sQ = base + L::kQ, sDO = base + L::kDO, sK = base + L::kK, sV = base + L::kV;
  auto bar = [&](int i) { return base + L::kBars + 8u * uint32_t(i); };
  volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(sbase + L::kTmemPtr);
  volatile int *abort = reinterpret_cast<volatile int *>(sbase + L::kAbort);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_items = int(p.status[kStFwdItems]);

  if (tid == 0) {
    mbar_init(bar(kDBarQFull), 1);
    mbar_init(bar(kDBarQEmpty), 1);
    for (int s = 0; s < kDStages; ++s) {
      mbar_init(bar(kDBarKFull + s), 1);
      mbar_init(bar(kDBarKEmpty + s), 1);
      mbar_init(bar(kDBarVFull + s), 1);
      mbar_init(bar(kDBarVEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(kDBarSFull + b), 1);
      mbar_init(bar(kDBarSFree + b), 1);
      mbar_init(bar(kDBarDSFull + b), kDSoftmaxThreads);
    }
    mbar_init(bar(kDBarDPFull), 1);
    mbar_init(bar(kDBarDPFree), kDSoftmaxThreads);
    mbar_init(bar(kDBarDQDone), 1);
    mbar_init(bar(kDBarDrain), 1);
    mbar_init(bar(kDBarDrainS), 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == kDQMmaWarp) {
    tmem_alloc(base + L::kTmemPtr, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS0 = tmem, tDP = tmem + 256u, tDQ = tmem + 384u;

  if (warp == kDLoadWarp || warp == kDVLoadWarp) {
    // ----------------------------------------------------- TMA producers
    const bool is_k = warp == kDLoadWarp;
    if (lane == 0) {
      const CUtensorMap *map = is_k ? &map_k : &map_v;
      if (is_k) {
        tma_prefetch_desc(&map_q);
        tma_prefetch_desc(&map_do);
      }
      tma_prefetch_desc(map);
      const uint32_t ring = is_k ? sK : sV;
      const int full0 = is_k ? kDBarKFull : kDBarVFull, empty0 = is_k ? kDBarKEmpty : kDBarVEmpty;
      uint32_t kv_it = 0, q_it = 0;
      int armed_q = -1, armed[kDStages] = {-1, -1};
      bool ok = true;
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        const ItemView v = item_view(p, p.fwd_items[it]);
        if (settle(p, v, Chunk{0, 0}).x >= v.ncnt) continue;  // no chunk: nothing to load
        if (is_k) {
          if (!(ok = wait_bar_lazy(bar(kDBarQEmpty), (q_it & 1u) ^ 1u, abort, p.status))) break;
          mbar_expect_tx(bar(kDBarQFull), 2 * L::kTile);
          armed_q = int(q_it & 1u);
          const int tok = p.q_layout == BSA_LAYOUT_TND ? int(v.bi.q_tok0) + v.t0 : v.t0;
          const int bb = p.q_layout == BSA_LAYOUT_TND ? 0 : v.b;
          tma_load_5d(sQ, &map_q, bar(kDBarQFull), 0, tok, 0, v.h1, bb);
          tma_load_5d(sDO, &map_do, bar(kDBarQFull), 0, tok, 0, v.h1, bb);
          ++q_it;
        }
        for (Chunk ch = settle(p, v, Chunk{0, 0}); ch.x < v.ncnt; ch = next_chunk(p, v, ch)) {
          const int s = int(kv_it % kDStages);
          const uint32_t ph = (kv_it / kDStages) & 1u;
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
            // the next item's Q and dOut tiles into L2 while this item ends
            const ItemView w = item_view(p, p.fwd_items[it + gridDim.x]);
            const int tok = p.q_layout == BSA_LAYOUT_TND ? int(w.bi.q_tok0) + w.t0 : w.t0;
            const int bb = p.q_layout == BSA_LAYOUT_TND ? 0 : w.b;
            tma_prefetch_l2_5d(&map_q, 0, tok, 0, w.h1, bb);
            tma_prefetch_l2_5d(&map_do, 0, tok, 0, w.h1, bb);
          }
          ++kv_it;
        }
      }
      if (*abort) {  // let every copy already issued land before the CTA exits
        if (armed_q >= 0) drain_wait(bar(kDBarQFull), uint32_t(armed_q));
        for (int s = 0; s < kDStages; ++s)
          if (armed[s] >= 0) drain_wait(bar(full0 + s), uint32_t(armed[s]));
      }
    }
  } else if (warp == kDQMmaWarp || warp == kDSMmaWarp) {
    // -------------------------------------------------------- MMA issuers
    // S and dP (SS form, both K-major over D) from warp 11; dQ (TS form,
    // dS from TMEM, K as the MN-major operand) from warp 9, on another
    // scheduler.  Each runs warp-uniform loops; one elected lane issues.
    constexpr uint32_t idS = idesc_f16(BF16, 128, 128, false, false);
    constexpr uint32_t idDQ = idesc_f16(BF16, 128, D, false, true);
    const uint64_t dQd = sw128_desc(sQ, 16, 1024);
    const uint64_t dOd = sw128_desc(sDO, 16, 1024);
    const uint64_t dKk = sw128_desc(sK, 16, 1024);
    const uint64_t dVk = sw128_desc(sV, 16, 1024);
    const uint64_t dKmn = sw128_desc(sK, L::kBox, 1024);
    auto kstep = [](int kk) { return uint64_t((kk >> 2) * (L::kBox >> 4) + (kk & 3) * 2); };
    // 16 kv columns of dS = 8 TMEM columns; the first 64 kv columns' dS is in
    // columns [0, 32) of the S buffer, the next 64's in [64, 96)
    auto pcol = [](int kk) { return uint32_t(64 * (kk >> 2) + 8 * (kk & 3)); };
    const bool is_s = warp == kDSMmaWarp;
    uint32_t kv_it = 0, q_it = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
      const ItemView v = item_view(p, p.fwd_items[it]);
      const int n = count_chunks_warp(p, v, lane);
      if (n == 0) continue;
      if (is_s) {
        if (!(ok = wait_warp(bar(kDBarQFull), q_it & 1u, abort, p.status))) break;
        ++q_it;
        for (int j = 0; j < n && ok; ++j) {
          const uint32_t t = kv_it + uint32_t(j);
          const int b = int(t & 1u), st = int(t % kDStages);
          // S_t reuses the buffer of dS_{t-2} once dQ_{t-2} is done
          if (t >= 2u && !(ok = wait_warp(bar(kDBarSFree + b), ((t >> 1) - 1u) & 1u, abort, p.status)))
            break;
          if (!(ok = wait_warp(bar(kDBarKFull + st), (t / kDStages) & 1u, abort, p.status))) break;
          tc_fence_after();
          const uint32_t da = tS0 + uint32_t(b) * 128u;
          const uint64_t ka = dKk + uint64_t(st * (L::kTile >> 4));
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) mma_ss_e(da, dQd + kstep(kk), ka + kstep(kk), idS, kk > 0 ? 1u : 0u);
          mma_commit_e(bar(kDBarSFull + b));
          // dP_t into the single dP buffer once every thread has read dP_{t-1}
          if (!(ok = wait_warp(bar(kDBarVFull + st), (t / kDStages) & 1u, abort, p.status))) break;
          if (t >= 1u && !(ok = wait_warp(bar(kDBarDPFree), (t - 1u) & 1u, abort, p.status))) break;
          tc_fence_after();
          const uint64_t va = dVk + uint64_t(st * (L::kTile >> 4));
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) mma_ss_e(tDP, dOd + kstep(kk), va + kstep(kk), idS, kk > 0 ? 1u : 0u);
          mma_commit_e(bar(kDBarDPFull));
          mma_commit_e(bar(kDBarVEmpty + st));
          if (j == n - 1) mma_commit_e(bar(kDBarQEmpty));
        }
      } else {
        for (int j = 0; j < n && ok; ++j) {
          const uint32_t t = kv_it + uint32_t(j);
          const int b = int(t & 1u), st = int(t % kDStages);
          // dS_t written (and, for a partial chunk, K_t's rows past the used
          // length zeroed by the softmax warps)
          if (!(ok = wait_warp(bar(kDBarDSFull + b), (t >> 1) & 1u, abort, p.status))) break;
          tc_fence_after();
          const uint32_t pa = tS0 + uint32_t(b) * 128u;
          const uint64_t kd = dKmn + uint64_t(st * (L::kTile >> 4));
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts_e(tDQ, pa + pcol(kk), kd + uint64_t(kk * 128), idDQ, (j == 0 && kk == 0) ? 0u : 1u);
          mma_commit_e(bar(kDBarSFree + b));
          mma_commit_e(bar(kDBarKEmpty + st));
          if (j == n - 1) mma_commit_e(bar(kDBarDQDone));
        }
      }
      kv_it += uint32_t(n);
    }
    if (*abort) {  // let issued MMAs finish before TMEM is freed
      const int dr = is_s ? kDBarDrainS : kDBarDrain;
      mma_commit_e(bar(dr));
      if (lane == 0) drain_wait(bar(dr), 0);
    }
    __syncwarp();
  } else if (warp < kDLoadWarp) {
    // ------------------------------------------------ the softmax groups
    const int wg = warp >> 2;
    const int r = tid & 127;  // query row = TMEM lane
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
    const float kLog2e = 1.4426950408889634f;
    uint32_t kv_it = 0, dq_it = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
      const ItemView v = item_view(p, p.fwd_items[it]);
      const bool live = r < v.rows;
      const int t = v.t0 + r;
      // lse (log2 units) and Dsum of this row; a row past qlen or with no
      // visible key gets lse = +inf, so its P and dS are 0
      float lse2 = INFINITY, dsum = 0.f;
      if (live) {
        const float l2 = p.lse[q_row(p.l_sb, p.l_sh, p.l_st, v.bi, v.b, v.h1, t)] * kLog2e;
        lse2 = l2 > -INFINITY ? l2 : INFINITY;
        const int64_t srow = p.q_layout == BSA_LAYOUT_BNSD ? int64_t(v.b) * p.Sq + t : v.bi.q_tok0 + t;
        dsum = p.dsum[srow * p.N1 + v.h1];
      }
      const int coff = kCausal ? t + v.kvlen - v.bi.qlen : 0;  // last kv token this row sees
      int n = 0;
      for (Cursor ck = cur_begin(p, v); ck.x < v.ncnt && ok; cur_next(p, v, ck), ++n, ++kv_it) {
        const int b = int(kv_it & 1u), st = int(kv_it % kDStages);
        if (!(ok = wait_warp(bar(kDBarSFull + b), (kv_it >> 1) & 1u, abort, p.status))) break;
        if (!(ok = wait_warp(bar(kDBarDPFull), kv_it & 1u, abort, p.status))) break;
        tc_fence_after();
        const int u0c = cur_u0(v, ck);
        const int valid_all = v.kvlen - u0c;  // kv columns of the chunk that exist
        const int vis_all = kCausal ? min(valid_all, coff - u0c + 1) : valid_all;
        const int valid = vis_all - 64 * wg;  // of this group's columns
        const uint32_t tS = tS0 + uint32_t(b) * 128u + lane_off;
        uint32_t dd[32];
        auto body = [&](auto masked) {
          // 16-column blocks of S and dP, the next block's loads in flight
          // while this one is computed
          const uint32_t c0 = uint32_t(64 * wg);
          uint32_t xs[2][16], xd[2][16];
          tmem_ld16(tS + c0, xs[0]);
          tmem_ld16(tDP + lane_off + c0, xd[0]);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            if (k + 1 < 4) {
              tmem_ld16(tS + c0 + uint32_t(16 * (k + 1)), xs[(k + 1) & 1]);
              tmem_ld16(tDP + lane_off + c0 + uint32_t(16 * (k + 1)), xd[(k + 1) & 1]);
            }
            const uint32_t *bs = xs[k & 1], *bd = xd[k & 1];
#pragma unroll
            for (int c2 = 0; c2 < 16; c2 += 2) {
              const int c = 16 * k + c2;
              // the pair's P and dS by paired fp32 operations (the same bits as
              // the scalar forms)
              const float2 a2 = fma2(make_float2(__uint_as_float(bs[c2]), __uint_as_float(bs[c2 + 1])),
                                     make_float2(p.scale_log2, p.scale_log2), make_float2(-lse2, -lse2));
              const float2 t2 = add2(make_float2(__uint_as_float(bd[c2]), __uint_as_float(bd[c2 + 1])),
                                     make_float2(-dsum, -dsum));
              const float2 s2 = mul2(make_float2(ex2(a2.x), ex2(a2.y)), t2);
              float s0 = s2.x, s1 = s2.y;
              if constexpr (decltype(masked)::value) {
                // columns past the used length or (causal) past the row's
                // last visible token: exactly 0, whatever S and dP hold there
                s0 = c < valid ? s0 : 0.f;
                s1 = c + 1 < valid ? s1 : 0.f;
              }
              dd[8 * k + (c2 >> 1)] = Pack2<T>::pack(s0, s1);
            }
            if (k + 1 < 4) tmem_wait_ld();
          }
        };
        if (__any_sync(0xffffffffu, valid < 64))
          body(std::true_type{});
        else
          body(std::false_type{});
        // every load of dP_t has completed (tmem_wait_ld): dP_{t+1} may go
        tc_fence_before();
        mbar_arrive(bar(kDBarDPFree));
        tmem_st32(tS + uint32_t(64 * wg), dd);
        if (valid_all < 128) {
          // kv rows past the used length may hold anything, even NaN; dQ
          // reads K_t, so zero those rows (their dS is already 0)
          uint4 *kt = reinterpret_cast<uint4 *>(sbase + L::kK + st * L::kTile);
          const int per_half = (128 - valid_all) * 8;  // 16-byte words per 64-column half
          for (int w = tid; w < per_half * (D / 64); w += kDSoftmaxThreads) {
            const int h = w / per_half, x = w % per_half;
            kt[h * (L::kBox / 16) + valid_all * 8 + x] = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(kDBarDSFull + b));
      }
      if (!ok) break;
      // ---- epilogue: dq = dtype(scale * dQ); group w writes D/2 columns,
      // stored through an in-warp transpose so that each store writes whole rows
      constexpr int kC = D / 16;  // 16-byte chunks of a thread's D/2 columns
      const int wrow = 32 * (warp & 3);  // this warp's first row of the tile
      uint4 qch[kC];
      if (n > 0) {
        if (!(ok = wait_warp(bar(kDBarDQDone), dq_it & 1u, abort, p.status))) break;
        ++dq_it;
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          uint32_t x[32];
          tmem_ld32(tDQ + lane_off + uint32_t((D / 2) * wg + 32 * h), x);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            qch[4 * h + c].x = Pack2<T>::pack(__uint_as_float(x[8 * c]) * p.scale, __uint_as_float(x[8 * c + 1]) * p.scale);
            qch[4 * h + c].y = Pack2<T>::pack(__uint_as_float(x[8 * c + 2]) * p.scale, __uint_as_float(x[8 * c + 3]) * p.scale);
            qch[4 * h + c].z = Pack2<T>::pack(__uint_as_float(x[8 * c + 4]) * p.scale, __uint_as_float(x[8 * c + 5]) * p.scale);
            qch[4 * h + c].w = Pack2<T>::pack(__uint_as_float(x[8 * c + 6]) * p.scale, __uint_as_float(x[8 * c + 7]) * p.scale);
          }
        }
      } else {
#pragma unroll
        for (int c = 0; c < kC; ++c) qch[c] = make_uint4(0, 0, 0, 0);
      }
      transpose_chunks<kC>(qch, lane);
      T *qrow0 = static_cast<T *>(p.dq) + q_row(p.dq_sb, p.dq_sh, p.dq_st, v.bi, v.b, v.h1, v.t0 + wrow) + (D / 2) * wg;
      store_rows<kC>(qrow0, p.dq_st, v.rows - wrow, qch, lane);
      // dQ is free for the next item once every softmax thread has arrived
      // on that item's first dS_full (the dQ issuer waits for it)
      tc_fence_before();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kDQMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, bool BF16, bool kCausal>
cudaError_t launch_dq(const Problem &p, const DqMaps &m, cudaStream_t s) {
  const int smem = DLayout<D>::kBytes > 120 * 1024 ? DLayout<D>::kBytes : 120 * 1024;
  cudaError_t e = cudaFuncSetAttribute(k_dq_tc<D, BF16, kCausal>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = p.fwd_slots < num_sms() ? p.fwd_slots : num_sms();
  if (grid <= 0) return cudaSuccess;
  e = launch_dep(k_dq_tc<D, BF16, kCausal>, dim3(unsigned(grid)), dim3(kDThreads), size_t(smem), s,
                 p, m.q, m.k, m.v, m.dout);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <bool kCausal>
cudaError_t launch_dq_for(const Problem &p, const DqMaps &m, cudaStream_t s) {
  if (p.dtype == BSA_BF16)
    return p.D == 64 ? launch_dq<64, true, kCausal>(p, m, s) : launch_dq<128, true, kCausal>(p, m, s);
  return p.D == 64 ? launch_dq<64, false, kCausal>(p, m, s) : launch_dq<128, false, kCausal>(p, m, s);
}

}  // namespace

cudaError_t launch_dq_main(const Problem &p, cudaStream_t s) {
  DqMaps m;
  cudaError_t e = make_dq_maps(p, m);
  if (e != cudaSuccess) return e;
  return p.causal ? launch_dq_for<true>(p, m, s) : launch_dq_for<false>(p, m, s);
}

}  // namespace bsa
