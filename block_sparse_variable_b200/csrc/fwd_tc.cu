// fwd_tc.cu -- tcgen05 / TMEM / TMA forward for sm_100a.
//
// Math (BlockSparseAttentionGrad README, "Formula"; BlitzSparseAttention,
// "softmax_lse output"): out = softmax(scale * Q K_sel^T) V_sel per query
// row over the kv tokens of the blocks in the row's compacted index row,
// lse = natural log of the sum of exp(scale * q.k).
//
// One persistent CTA per SM; each work item is 128 query rows of one head.
// Warp roles (256 threads):
//   warp 0      TMA producer: Q tile once per item, then K and V 128-row
//               chunks of the selected kv blocks into a 2-stage ring.
//   warp 1      TMEM owner and MMA issuer (one elected lane):
//                 S_j = Q K_j^T        (SS form, fp32 accumulator in TMEM)
//                 O  += P_j V_j        (TS form, P read from TMEM)
//   warps 4..7  softmax warpgroup, one query row per thread (TMEM lane):
//               reads S_j, masks kv columns past kvlen, keeps the running
//               max m (log2 domain) and sum l, writes P_j = exp2(s - m)
//               as packed 16-bit pairs back over S_j, and rescales O only
//               when the running max grew by more than 2^8 (so P stays
//               below 256); epilogue O / l and lse = (m + log2 l) ln 2.
// S is double-buffered in TMEM so S_{j+1} = Q K_{j+1}^T runs on the tensor
// cores while the softmax warpgroup works on S_j.
// TMEM columns: [0,128) S buffer 0, [128,256) S buffer 1, [256,256+D) O.
// Every wait on an mbarrier is bounded; on expiry the CTA raises
// BSA_FLAG_TIMEOUT, drains its in-flight copies and MMAs, frees TMEM and
// returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>

#include "addr.cuh"
#include "bsa_internal.h"
#include "ptx_sm80.cuh"
#include "sm100.cuh"
#include "tc_common.h"

namespace bsa {
namespace {

using namespace sm100;

constexpr int kTcThreads = 384;
constexpr int kStages = 2;
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s: any legitimate wait is far shorter
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when m grows by > 2^8

// barrier slots
enum : int {
  kBarQFull = 0,
  kBarQEmpty = 1,
  kBarKFull = 2,   // + stage
  kBarKEmpty = 4,  // + stage
  kBarVFull = 6,   // + stage
  kBarVEmpty = 8,  // + stage
  kBarSFull = 10,  // + buffer
  kBarPFull = 12,  // + buffer
  kBarPVDone = 14,  // + (chunk index % 2): P_t V_t is in O
  kBarDrain = 16,
  kNumBars = 17
};

template <int D>
struct Layout {
  static constexpr int kBox = 128 * 128;              // one 128-row x 64-col 16-bit box
  static constexpr int kTile = (D / 64) * kBox;       // Q / K / V tile
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTile;
  static constexpr int kV = kK + kStages * kTile;
  static constexpr int kBars = kV + kStages * kTile;
  static constexpr int kXchg = kBars + kNumBars * 8 + 8;  // [2][2][128] floats (max, sum)
  static constexpr int kTmemPtr = kXchg + 2 * 2 * 128 * 4;
  static constexpr int kAbort = kTmemPtr + 4;
  static constexpr int kBytes = kAbort + 4;
  static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024
};

struct Chunk {
  int x, c;  // compacted-row position, 128-row chunk of that kv block
};

// every role walks the same chunk sequence of an item
struct ItemView {
  int b, h1, h2, t0, rows, kvlen, ncnt, ksl, BKV;
  const uint16_t *crow;
  BatchInfo bi;
  __device__ int u0(const Chunk &ch) const { return int(crow[ch.x]) * BKV + ch.c * 128; }
};

__device__ __forceinline__ bool page_ok(const Problem &p, const ItemView &v, int u0, int &pg) {
  if (p.kv_layout != BSA_LAYOUT_PA_BBND) { pg = 0; return true; }
  pg = kv_page(p, v.b, u0);
  return pg >= 0;
}

__device__ __forceinline__ Chunk settle(const Problem &p, const ItemView &v, Chunk ch) {
  int pg;
  while (ch.x < v.ncnt && !page_ok(p, v, v.u0(ch), pg)) {
    ++ch.c;
    if (ch.c >= v.ksl || v.u0(ch) >= v.kvlen) { ++ch.x; ch.c = 0; }
  }
  return ch;
}
__device__ __forceinline__ Chunk next_chunk(const Problem &p, const ItemView &v, Chunk ch) {
  ++ch.c;
  if (ch.c >= v.ksl || v.u0(ch) >= v.kvlen) { ++ch.x; ch.c = 0; }
  return settle(p, v, ch);
}
__device__ __forceinline__ int count_chunks(const Problem &p, const ItemView &v) {
  int n = 0;
  for (Chunk ch = settle(p, v, Chunk{0, 0}); ch.x < v.ncnt; ch = next_chunk(p, v, ch)) ++n;
  return n;
}

__device__ __forceinline__ ItemView item_view(const Problem &p, int id) {
  ItemView v;
  const int qs = id % p.nsub;
  const int gq = (id / p.nsub) % p.Rg;
  v.h1 = id / (p.nsub * p.Rg);
  v.b = p.row_batch[gq];
  v.bi = p.batch[v.b];
  const int i = gq - v.bi.qoff;
  v.t0 = i * p.BQ + qs * 128;
  v.rows = min(128, v.bi.qlen - v.t0);
  v.h2 = v.h1 / p.g;
  const int hi = p.Hidx == p.N1 ? v.h1 : v.h2;
  const int64_t ci = int64_t(hi) * p.Rg + gq;
  v.crow = p.comp + ci * p.W;
  v.ncnt = p.ncomp[ci];
  v.kvlen = v.bi.kvlen;
  v.ksl = p.ksl;
  v.BKV = p.BKV;
  return v;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait: gives up after kWaitNs of wall time (raising the abort flag
// and BSA_FLAG_TIMEOUT), or as soon as another role has aborted.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int *abort,
                                         uint32_t *status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0u) {
      if (*abort) return false;
      if (global_ns() - t0 > kWaitNs) {
        *abort = 1;
        atomicOr(status + kStFlags, BSA_FLAG_TIMEOUT);
        return false;
      }
    }
  }
}

// the same, agreed by the whole warp (tcgen05 .sync.aligned ops follow)
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, volatile int *abort,
                                          uint32_t *status) {
  const bool r = wait_bar(bar, parity, abort, status);
  return __all_sync(0xffffffffu, r);
}

__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(threads) : "memory");
}

// drain wait on the abort path: bounded, result ignored
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity) && global_ns() - t0 < kWaitNs) {
  }
}

template <int D, bool BF16>
__global__ void __launch_bounds__(kTcThreads, 1)
    k_fwd_tc(const Problem p, const __grid_constant__ CUtensorMap map_q,
             const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v) {
  using L = Layout<D>;
  using T = typename std::conditional<BF16, __nv_bfloat16, __half>::type;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  unsigned char *sbase = smem_raw + (base - raw_base);
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
      mbar_init(bar(kBarSFull + s), 1);
      mbar_init(bar(kBarPFull + s), 128);
    }
    mbar_init(bar(kBarPVDone), 1);
    mbar_init(bar(kBarPVDone + 1), 1);
    mbar_init(bar(kBarDrain), 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(base + L::kTmemPtr, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS0 = tmem, tO0 = tmem + 256;  // S_w at tS0 + 128w, O_w at tO0 + D*w

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      uint32_t kv_it = 0, q_it = 0;
      int armed_q = -1, armed_k[kStages] = {-1, -1}, armed_v[kStages] = {-1, -1};
      bool ok = true;
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
        const ItemView v = item_view(p, p.fwd_items[it]);
        if (count_chunks(p, v) == 0) continue;
        ok = wait_bar(bar(kBarQEmpty), (q_it & 1u) ^ 1u, abort, p.status);
        if (!ok) break;
        mbar_expect_tx(bar(kBarQFull), L::kTile);
        armed_q = int(q_it & 1u);
        {
          const int tok = p.q_layout == BSA_LAYOUT_TND ? int(v.bi.q_tok0) + v.t0 : v.t0;
          const int bb = p.q_layout == BSA_LAYOUT_TND ? 0 : v.b;
          for (int h = 0; h < D / 64; ++h)
            tma_load_4d(sQ + h * L::kBox, &map_q, bar(kBarQFull), h * 64, tok, v.h1, bb);
        }
        ++q_it;
        for (Chunk ch = settle(p, v, Chunk{0, 0}); ch.x < v.ncnt; ch = next_chunk(p, v, ch)) {
          const int s = int(kv_it % kStages);
          const uint32_t ph = (kv_it / kStages) & 1u;
          const int u0 = v.u0(ch);
          int pg;
          page_ok(p, v, u0, pg);
          int c1, c2, c3;  // coordinates after the head-dim one
          if (p.kv_layout == BSA_LAYOUT_PA_BBND) { c1 = v.h2; c2 = u0 % p.page_size; c3 = pg; }
          else if (p.kv_layout == BSA_LAYOUT_TND) { c1 = int(v.bi.kv_tok0) + u0; c2 = v.h2; c3 = 0; }
          else { c1 = u0; c2 = v.h2; c3 = v.b; }
          if (!(ok = wait_bar(bar(kBarKEmpty + s), ph ^ 1u, abort, p.status))) break;
          mbar_expect_tx(bar(kBarKFull + s), L::kTile);
          armed_k[s] = int(ph);
          for (int h = 0; h < D / 64; ++h)
            tma_load_4d(sK + s * L::kTile + h * L::kBox, &map_k, bar(kBarKFull + s), h * 64, c1, c2, c3);
          if (!(ok = wait_bar(bar(kBarVEmpty + s), ph ^ 1u, abort, p.status))) break;
          mbar_expect_tx(bar(kBarVFull + s), L::kTile);
          armed_v[s] = int(ph);
          for (int h = 0; h < D / 64; ++h)
            tma_load_4d(sV + s * L::kTile + h * L::kBox, &map_v, bar(kBarVFull + s), h * 64, c1, c2, c3);
          ++kv_it;
        }
      }
      if (*abort) {  // let every copy already issued land before the CTA exits
        if (armed_q >= 0) drain_wait(bar(kBarQFull), uint32_t(armed_q));
        for (int s = 0; s < kStages; ++s) {
          if (armed_k[s] >= 0) drain_wait(bar(kBarKFull + s), uint32_t(armed_k[s]));
          if (armed_v[s] >= 0) drain_wait(bar(kBarVFull + s), uint32_t(armed_v[s]));
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    constexpr uint32_t idS = idesc_f16(BF16, 128, 128, false, false);
    constexpr uint32_t idPV = idesc_f16(BF16, 128, D, false, true);
    uint32_t kv_it = 0, q_it = 0;
    bool ok = true;
    auto issue_pv = [&](uint32_t t, bool first, int valid) {
      const int s = int(t % kStages);
      const uint32_t ph = (t / kStages) & 1u;
      if (!(ok = wait_warp(bar(kBarPFull + s), ph, abort, p.status))) return;
      if (!(ok = wait_warp(bar(kBarVFull + s), ph, abort, p.status))) return;
      if (p.kv_layout == BSA_LAYOUT_PA_BBND && valid < 128) {
        // rows of the last page past the used length may hold anything
        // (even NaN); their P is 0, so make their V exactly 0 as well
        uint4 *vt = reinterpret_cast<uint4 *>(sbase + L::kV + s * L::kTile);
        const int per_half = (128 - valid) * 8;  // 16-byte words per 64-column half
        for (int w = lane; w < per_half * (D / 64); w += 32) {
          const int h = w / per_half, x = w % per_half;
          vt[h * (L::kBox / 16) + valid * 8 + x] = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t a_tmem = tS0 + uint32_t(s) * 128u;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bdesc = sw128_desc(sV + s * L::kTile + kk * 2048, L::kBox, 1024);
          mma_ts(tO0 + uint32_t(s) * D, a_tmem + uint32_t(kk) * 8u, bdesc, idPV,
                 (first && kk == 0) ? 0u : 1u);
        }
        mma_commit(bar(kBarPVDone + s));
        mma_commit(bar(kBarVEmpty + s));
      }
      __syncwarp();
    };
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
      const ItemView v = item_view(p, p.fwd_items[it]);
      const int n = count_chunks(p, v);
      if (n == 0) continue;
      if (!(ok = wait_warp(bar(kBarQFull), q_it & 1u, abort, p.status))) break;
      ++q_it;
      int prev_valid = 128;
      Chunk ch = settle(p, v, Chunk{0, 0});
      for (int j = 0; j < n && ok; ++j) {
        const int s = int(kv_it % kStages);
        const uint32_t ph = (kv_it / kStages) & 1u;
        if (!(ok = wait_warp(bar(kBarKFull + s), ph, abort, p.status))) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t d_tmem = tS0 + uint32_t(s) * 128u;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = uint32_t(kk >> 2) * L::kBox + uint32_t(kk & 3) * 32u;
            mma_ss(d_tmem, sw128_desc(sQ + off, 16, 1024),
                   sw128_desc(sK + s * L::kTile + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(kBarSFull + s));
          mma_commit(bar(kBarKEmpty + s));
          if (j == n - 1) mma_commit(bar(kBarQEmpty));
        }
        __syncwarp();
        if (j >= 1) issue_pv(kv_it - 1, j <= 2, prev_valid);
        prev_valid = v.kvlen - v.u0(ch);
        ch = next_chunk(p, v, ch);
        ++kv_it;
      }
      if (ok) issue_pv(kv_it - 1, n <= 2, prev_valid);
    }
    if (*abort && lane == 0) {  // let issued MMAs finish before TMEM is freed
      mma_commit(bar(kBarDrain));
      drain_wait(bar(kBarDrain), 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------- two softmax warpgroups
    // Warpgroup w takes the chunks whose global index t has t % 2 == w: its
    // own S buffer, O accumulator, running max and sum (a split of the kv
    // range inside the CTA); the halves are merged in the epilogue.
    const int wg = (warp - 4) >> 2;
    const int r = (tid - 128) & 127;                        // query row = TMEM lane
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tS = tS0 + uint32_t(wg) * 128u + lane_off;
    const uint32_t tOw = tO0 + uint32_t(wg) * D + lane_off;
    float *xm = reinterpret_cast<float *>(sbase + L::kXchg);  // [2][128] max
    float *xl = xm + 256;                                     // [2][128] sum
    const float kLn2 = 0.6931471805599453f;
    uint32_t kv_it = 0, own = 0;  // global chunk counter; chunks this group took
    bool ok = true;
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
      const ItemView v = item_view(p, p.fwd_items[it]);
      float m = -INFINITY, l = 0.f;
      int n = 0;
      for (Chunk ch = settle(p, v, Chunk{0, 0}); ch.x < v.ncnt && ok;
           ch = next_chunk(p, v, ch), ++n, ++kv_it) {
        if (int(kv_it & 1u) != wg) continue;
        if (!(ok = wait_warp(bar(kBarSFull + wg), own & 1u, abort, p.status))) break;
        tc_fence_after();
        const int valid = v.kvlen - v.u0(ch);  // kv columns of this chunk that exist
        // the whole 128-column row in one round trip
        uint32_t x[4][32];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld32(tS + uint32_t(q) * 32u, x[q]);
        tmem_wait_ld();
        if (valid < 128) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (q * 32 + c >= valid) x[q][c] = __float_as_uint(-INFINITY);
        }
        float pm[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) pm[k] = -INFINITY;
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int c = 0; c < 32; ++c) pm[c & 7] = fmaxf(pm[c & 7], __uint_as_float(x[q][c]));
        const float cmax = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                                 fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7]))) * p.scale_log2;
        // running max: adopted on the group's first chunk; afterwards kept
        // stale until it falls more than 2^8 behind (then O and l rescale)
        const bool first = m == -INFINITY;
        const bool grow = __any_sync(0xffffffffu, !first && cmax > m + kRescaleThreshold);
        const float m_new = first ? cmax : (grow ? fmaxf(m, cmax) : m);
        const float alpha = (first || !grow) ? 1.f : ex2(m - m_new);
        m = m_new;
        // P = exp2(scale*log2(e)*s - m), written over S as 16-bit pairs
        float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[32];
#pragma unroll
          for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              const float e0 = ex2(fmaf(__uint_as_float(x[2 * h + q][c]), p.scale_log2, -m));
              const float e1 = ex2(fmaf(__uint_as_float(x[2 * h + q][c + 1]), p.scale_log2, -m));
              ps[(c >> 1) & 3] += e0 + e1;
              pk[q * 16 + (c >> 1)] = MmaOp<T>::pack(e0, e1);
            }
          tmem_st32(tS + uint32_t(h) * 32u, pk);
        }
        l = l * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
        if (grow) {
          // O may only be rescaled once this group's previous P V (t - 2,
          // same accumulator) has landed in it
          const uint32_t t = kv_it - 2;
          if (!(ok = wait_warp(bar(kBarPVDone + wg), (t / 2) & 1u, abort, p.status))) break;
          tc_fence_after();
#pragma unroll
          for (int q = 0; q < D / 32; ++q) {
            uint32_t o[32];
            tmem_ld32(tOw + uint32_t(q) * 32u, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(tOw + uint32_t(q) * 32u, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(kBarPFull + wg));
        ++own;
      }
      if (!ok) break;
      // ---- epilogue: merge the two groups' partial results
      const bool live = r < v.rows;
      T *orow = static_cast<T *>(p.out) + q_row(p.o_sb, p.o_sh, p.o_st, v.bi, v.b, v.h1, v.t0 + r);
      if (n > 0) {
        const uint32_t t = kv_it - 1;  // the item's last P V; earlier ones precede it
        if (!(ok = wait_warp(bar(kBarPVDone + int(t & 1u)), (t / 2) & 1u, abort, p.status))) break;
        tc_fence_after();
      }
      xm[wg * 128 + r] = m;
      xl[wg * 128 + r] = l;
      named_sync(1, 256);
      const float m0 = xm[r], m1 = xm[128 + r], l0 = xl[r], l1 = xl[128 + r];
      const float M = fmaxf(m0, m1);
      const float a0 = m0 == -INFINITY ? 0.f : ex2(m0 - M);
      const float a1 = m1 == -INFINITY ? 0.f : ex2(m1 - M);
      const float Lsum = l0 * a0 + l1 * a1;
      const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
      // group w writes columns [w*D/2, (w+1)*D/2) from both accumulators
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        const uint32_t col = uint32_t(wg) * (D / 2) + uint32_t(q) * 16u;
        uint32_t o0[16], o1[16];
        tmem_ld16(tO0 + lane_off + col, o0);
        tmem_ld16(tO0 + uint32_t(D) + lane_off + col, o1);
        tmem_wait_ld();
        if (live) {
          uint4 w[2];
          uint32_t *wp = reinterpret_cast<uint32_t *>(w);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float y0 = (a0 > 0.f ? __uint_as_float(o0[2 * c]) * a0 : 0.f) +
                             (a1 > 0.f ? __uint_as_float(o1[2 * c]) * a1 : 0.f);
            const float y1 = (a0 > 0.f ? __uint_as_float(o0[2 * c + 1]) * a0 : 0.f) +
                             (a1 > 0.f ? __uint_as_float(o1[2 * c + 1]) * a1 : 0.f);
            wp[c] = MmaOp<T>::pack(y0 * inv, y1 * inv);
          }
          reinterpret_cast<uint4 *>(orow + col)[0] = w[0];
          reinterpret_cast<uint4 *>(orow + col)[1] = w[1];
        }
      }
      if (wg == 0 && live && p.lse)
        p.lse[q_row(p.l_sb, p.l_sh, p.l_st, v.bi, v.b, v.h1, v.t0 + r)] =
            Lsum > 0.f ? (M + __log2f(Lsum)) * kLn2 : -INFINITY;
      tc_fence_before();
      named_sync(1, 256);  // both groups are done with O and the exchange slots
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, bool BF16>
cudaError_t launch_tc(const Problem &p, const FwdMaps &m, cudaStream_t s) {
  // at least 120 KB so that exactly one CTA (the sole owner of all 512 TMEM
  // columns) is resident per SM
  const int smem = Layout<D>::kAlloc > 120 * 1024 ? Layout<D>::kAlloc : 120 * 1024;
  cudaError_t e = cudaFuncSetAttribute(k_fwd_tc<D, BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = p.fwd_slots < num_sms() ? p.fwd_slots : num_sms();
  if (grid <= 0) return cudaSuccess;
  k_fwd_tc<D, BF16><<<unsigned(grid), kTcThreads, smem, s>>>(p, m.q, m.k, m.v);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_main(const Problem &p, cudaStream_t s) {
  FwdMaps m;
  cudaError_t e = make_fwd_maps(p, m);
  if (e != cudaSuccess) return e;
  if (p.dtype == BSA_BF16)
    return p.D == 64 ? launch_tc<64, true>(p, m, s) : launch_tc<128, true>(p, m, s);
  return p.D == 64 ? launch_tc<64, false>(p, m, s) : launch_tc<128, false>(p, m, s);
}

}  // namespace bsa
