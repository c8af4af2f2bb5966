// fwd_mma.cu -- register-tile forward (mma.sync m16n8k16, fp32 online
// softmax).  One CTA of 8 warps per 128-row query slice; persistent CTAs
// take items from the longest-first work list through an atomic counter.
// Each warp owns 16 query rows; K/V stream through shared memory in 64-row
// tiles (double-buffered cp.async), visiting only the kv blocks of the
// compacted index row.
//
// Math (BlockSparseAttentionGrad README, "Formula"; BlitzSparseAttention,
// "softmax_lse output"): per row, m = running max of scale*s, l = running
// sum of exp(scale*s - m) with rescaling, O = sum exp(scale*s - m) v;
// out = O / l, lse = m + ln l.  Scores of kv tokens at or past kvlen are
// -inf; a row with no selected token gets out 0 and lse -inf.
#include <cuda_runtime.h>

#include <cmath>

#include "addr.cuh"
#include "bsa_internal.h"
#include "ptx_sm80.cuh"

namespace bsa {
namespace {

constexpr int kFwdBM = 128;  // query rows per item
constexpr int kFwdBN = 64;   // kv rows per tile
constexpr int kFwdThreads = 256;

struct TileCursor {
  int x;  // position in the compacted index row
  int s;  // 64-row tile inside the kv block
};

template <int D, typename T>
__global__ void __launch_bounds__(kFwdThreads, 1) k_fwd_mma(const Problem p) {
  using Op = MmaOp<T>;
  constexpr int BM = kFwdBM, BN = kFwdBN, CH = D / 8;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  T *sQ = reinterpret_cast<T *>(smem_raw);
  T *sK = sQ + BM * D;
  T *sV = sK + 2 * BN * D;
  __shared__ int s_item;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int n_items = int(p.status[kStFwdItems]);
  const int tiles_per_block = p.BKV / BN;
  const float kLn2 = 0.6931471805599453f;

  for (;;) {
    if (tid == 0) s_item = int(atomicAdd(p.status + kStFwdNext, 1u));
    __syncthreads();
    const int it = s_item;
    if (it >= n_items) break;
    const int id = p.fwd_items[it];
    const int qs = id % p.nsub;
    const int gq = (id / p.nsub) % p.Rg;
    const int h1 = id / (p.nsub * p.Rg);
    const int b = p.row_batch[gq];
    const BatchInfo bi = p.batch[b];
    const int i = gq - bi.qoff;
    const int t0 = i * p.BQ + qs * kSlice;
    const int rows = min(BM, bi.qlen - t0);
    const int h2 = h1 / p.g;
    const int hi = p.Hidx == p.N1 ? h1 : h2;
    const int64_t crow_i = int64_t(hi) * p.Rg + gq;
    const uint16_t *crow = p.comp + crow_i * p.W;
    const int ncnt = p.ncomp[crow_i];
    const int kvlen = bi.kvlen;

    const T *qg = static_cast<const T *>(p.q);
    const T *kg = static_cast<const T *>(p.k);
    const T *vg = static_cast<const T *>(p.v);

    // ---- Q slice -> shared (rows past qlen are zero)
    for (int c = tid; c < BM * CH; c += kFwdThreads) {
      const int r = c / CH, ch = c % CH;
      const bool ok = r < rows;
      const T *src = qg + q_row(p.q_sb, p.q_sh, p.q_st, bi, b, h1, t0 + (ok ? r : 0)) + ch * 8;
      cp_async16(smem_u32(sQ + swz<D>(r, ch * 8)), src, ok ? 16 : 0);
    }

    // tile cursor helpers (uniform across the CTA)
    auto tile_start = [&](const TileCursor &c) { return int(crow[c.x]) * p.BKV + c.s * BN; };
    auto page_of = [&](int u0) {
      return p.kv_layout == BSA_LAYOUT_PA_BBND ? kv_page(p, b, u0) : 0;
    };
    auto settle = [&](TileCursor c) {  // skip tiles whose page is invalid
      while (c.x < ncnt && page_of(tile_start(c)) < 0) {
        if (tid == 0) atomicOr(p.status + kStFlags, BSA_FLAG_BAD_PAGE);
        ++c.s;
        if (c.s >= tiles_per_block || tile_start(c) >= kvlen) { ++c.x; c.s = 0; }
      }
      return c;
    };
    auto advance = [&](TileCursor c) {
      ++c.s;
      if (c.s >= tiles_per_block || tile_start(c) >= kvlen) { ++c.x; c.s = 0; }
      return settle(c);
    };
    auto load_kv = [&](int buf, const TileCursor &c) {
      const int u0 = tile_start(c);
      const int pg = page_of(u0);
      T *dk = sK + buf * BN * D;
      T *dv = sV + buf * BN * D;
      for (int x = tid; x < BN * CH; x += kFwdThreads) {
        const int r = x / CH, ch = x % CH;
        const bool ok = u0 + r < kvlen;
        const int u = ok ? u0 + r : u0;
        const int64_t ko = kv_row(p, p.k_sb, p.k_sh, p.k_st, bi, b, h2, u, pg) + ch * 8;
        const int64_t vo = kv_row(p, p.v_sb, p.v_sh, p.v_st, bi, b, h2, u, pg) + ch * 8;
        cp_async16(smem_u32(dk + swz<D>(r, ch * 8)), kg + ko, ok ? 16 : 0);
        cp_async16(smem_u32(dv + swz<D>(r, ch * 8)), vg + vo, ok ? 16 : 0);
      }
    };

    TileCursor cur = settle(TileCursor{0, 0});
    if (cur.x < ncnt) load_kv(0, cur);
    cp_async_commit();

    float o[D / 8][4];
#pragma unroll
    for (int d = 0; d < D / 8; ++d) o[d][0] = o[d][1] = o[d][2] = o[d][3] = 0.f;
    float m2[2] = {-INFINITY, -INFINITY};  // running max of scale*log2(e)*s
    float l[2] = {0.f, 0.f};
    uint32_t qf[D / 16][4];
    bool have_q = false;
    int buf = 0;

    while (cur.x < ncnt) {
      const TileCursor nxt = advance(cur);
      if (nxt.x < ncnt) load_kv(buf ^ 1, nxt);
      cp_async_commit();
      cp_async_wait<1>();
      __syncthreads();
      if (!have_q) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int r = warp * 16 + (lane & 15), c = kk * 16 + (lane >> 4) * 8;
          ldsm_x4(smem_u32(sQ + swz<D>(r, c)), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
        }
        have_q = true;
      }
      const T *Kt = sK + buf * BN * D;
      const T *Vt = sV + buf * BN * D;
      const int u0 = tile_start(cur);

      // S = Q K^T for this warp's 16 rows x 64 kv columns
      float s[BN / 8][4];
#pragma unroll
      for (int n = 0; n < BN / 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
        for (int np = 0; np < BN / 16; ++np) {
          const int r = np * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int c = kk * 16 + ((lane >> 3) & 1) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm_x4(smem_u32(Kt + swz<D>(r, c)), b0, b1, b2, b3);
          Op::run(s[2 * np], qf[kk], b0, b1);
          Op::run(s[2 * np + 1], qf[kk], b2, b3);
        }
      }
      if (u0 + BN > kvlen) {
#pragma unroll
        for (int n = 0; n < BN / 8; ++n) {
          const int u = u0 + n * 8 + 2 * t4;
          if (u >= kvlen) { s[n][0] = -INFINITY; s[n][2] = -INFINITY; }
          if (u + 1 >= kvlen) { s[n][1] = -INFINITY; s[n][3] = -INFINITY; }
        }
      }
      // online softmax (two rows per thread: g8 and g8 + 8)
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int n = 0; n < BN / 8; ++n) {
        mx0 = fmaxf(mx0, fmaxf(s[n][0], s[n][1]));
        mx1 = fmaxf(mx1, fmaxf(s[n][2], s[n][3]));
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m2[0], mx0 * p.scale_log2);
      const float mn1 = fmaxf(m2[1], mx1 * p.scale_log2);
      const float base0 = mn0 == -INFINITY ? 0.f : mn0;
      const float base1 = mn1 == -INFINITY ? 0.f : mn1;
      const float a0 = ex2(m2[0] - base0), a1 = ex2(m2[1] - base1);
      m2[0] = mn0;
      m2[1] = mn1;
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int n = 0; n < BN / 8; ++n) {
        s[n][0] = ex2(fmaf(s[n][0], p.scale_log2, -base0));
        s[n][1] = ex2(fmaf(s[n][1], p.scale_log2, -base0));
        s[n][2] = ex2(fmaf(s[n][2], p.scale_log2, -base1));
        s[n][3] = ex2(fmaf(s[n][3], p.scale_log2, -base1));
        rs0 += s[n][0] + s[n][1];
        rs1 += s[n][2] + s[n][3];
      }
      l[0] = l[0] * a0 + rs0;
      l[1] = l[1] * a1 + rs1;
#pragma unroll
      for (int d = 0; d < D / 8; ++d) {
        o[d][0] *= a0; o[d][1] *= a0;
        o[d][2] *= a1; o[d][3] *= a1;
      }
      // O += P V  (P rounded to the input dtype, the accumulator layout reused as A)
#pragma unroll
      for (int kk = 0; kk < BN / 16; ++kk) {
        uint32_t pa[4];
        pa[0] = Op::pack(s[2 * kk][0], s[2 * kk][1]);
        pa[1] = Op::pack(s[2 * kk][2], s[2 * kk][3]);
        pa[2] = Op::pack(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        pa[3] = Op::pack(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
        for (int dp = 0; dp < D / 16; ++dp) {
          const int r = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int c = dp * 16 + (lane >> 4) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(smem_u32(Vt + swz<D>(r, c)), b0, b1, b2, b3);
          Op::run(o[2 * dp], pa, b0, b1);
          Op::run(o[2 * dp + 1], pa, b2, b3);
        }
      }
      __syncthreads();
      cur = nxt;
      buf ^= 1;
    }
    cp_async_wait<0>();
    __syncthreads();

    // ---- epilogue: normalise, stage through shared, coalesced stores
    float ls0 = l[0] + __shfl_xor_sync(0xffffffffu, l[0], 1);
    ls0 += __shfl_xor_sync(0xffffffffu, ls0, 2);
    float ls1 = l[1] + __shfl_xor_sync(0xffffffffu, l[1], 1);
    ls1 += __shfl_xor_sync(0xffffffffu, ls1, 2);
    const float inv0 = ls0 > 0.f ? 1.f / ls0 : 0.f;
    const float inv1 = ls1 > 0.f ? 1.f / ls1 : 0.f;
    const int r0 = warp * 16 + g8, r1 = r0 + 8;
#pragma unroll
    for (int d = 0; d < D / 8; ++d) {
      *reinterpret_cast<uint32_t *>(sQ + swz<D>(r0, d * 8 + 2 * t4)) =
          Op::pack(o[d][0] * inv0, o[d][1] * inv0);
      *reinterpret_cast<uint32_t *>(sQ + swz<D>(r1, d * 8 + 2 * t4)) =
          Op::pack(o[d][2] * inv1, o[d][3] * inv1);
    }
    if (p.lse != nullptr && t4 == 0) {
      if (r0 < rows)
        p.lse[q_row(p.l_sb, p.l_sh, p.l_st, bi, b, h1, t0 + r0)] =
            ls0 > 0.f ? m2[0] * kLn2 + logf(ls0) : -INFINITY;
      if (r1 < rows)
        p.lse[q_row(p.l_sb, p.l_sh, p.l_st, bi, b, h1, t0 + r1)] =
            ls1 > 0.f ? m2[1] * kLn2 + logf(ls1) : -INFINITY;
    }
    __syncthreads();
    T *og = static_cast<T *>(p.out);
    for (int c = tid; c < BM * CH; c += kFwdThreads) {
      const int r = c / CH, ch = c % CH;
      if (r < rows)
        *reinterpret_cast<uint4 *>(og + q_row(p.o_sb, p.o_sh, p.o_st, bi, b, h1, t0 + r) + ch * 8) =
            *reinterpret_cast<const uint4 *>(sQ + swz<D>(r, ch * 8));
    }
    __syncthreads();
  }
}

template <int D, typename T>
cudaError_t launch_fwd_t(const Problem &p, cudaStream_t s) {
  const int smem = (kFwdBM * D + 4 * kFwdBN * D) * int(sizeof(T));
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(k_fwd_mma<D, T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int64_t grid = p.fwd_slots < num_sms() ? p.fwd_slots : num_sms();
  if (grid <= 0) return cudaSuccess;
  k_fwd_mma<D, T><<<unsigned(grid), kFwdThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_main(const Problem &p, cudaStream_t s) {
  if (p.dtype == BSA_BF16)
    return p.D == 64 ? launch_fwd_t<64, __nv_bfloat16>(p, s) : launch_fwd_t<128, __nv_bfloat16>(p, s);
  return p.D == 64 ? launch_fwd_t<64, __half>(p, s) : launch_fwd_t<128, __half>(p, s);
}

}  // namespace bsa
