// bwd_mma.cu -- register-tile backward (mma.sync m16n8k16).
//
// BlockSparseAttentionGrad README, "Formula", in the stage order of the
// aclnnFlashAttentionUnpaddingScoreGradV2 article, section 8.3 (recompute p,
// dp, ds, dq, dk, dv):
//   pre:   Dsum_t = sum_d dOut[t,d] * out[t,d]            (softmax_grad)
//   main:  one CTA per 128 kv rows of kv head h2 (KV-major, driven by the
//          inverted index); K, V stay in shared memory, dK, dV in registers.
//          For every q head of the GQA group and every query block that
//          selected this kv block, in 64-row query steps:
//            S^T = K Q^T,  P^T = exp(scale*S^T - lse)     (recompute p)
//            dP^T = V dOut^T                               (dp)
//            dS^T = P^T o (dP^T - Dsum)                    (ds)
//            dQacc[q rows] += dS K  (fp32 atomics)         (dq)
//            dK += dS^T Q,  dV += P^T dOut                 (dk, dv)
//          epilogue: dK *= scale; rows past kvlen stay 0.
//   post:  dq = dtype(scale * dQacc); zeros for kv rows no item covers.
#include <cuda_runtime.h>

#include <cmath>

#include "addr.cuh"
#include "bsa_internal.h"
#include "ptx_sm80.cuh"

namespace bsa {
namespace {

constexpr int kBwdBN = 128;  // kv rows per item
constexpr int kBwdBM = 64;   // query rows per step
constexpr int kBwdThreads = 256;

// q storage row r -> (batch, batch-local token) for the q-layout tensors
__device__ __forceinline__ int64_t qstore_off(const Problem &p, int64_t sb, int64_t sh, int64_t st,
                                              int64_t r, int h) {
  if (p.q_layout == BSA_LAYOUT_BNSD) return (r / p.Sq) * sb + (r % p.Sq) * st + int64_t(h) * sh;
  return r * st + int64_t(h) * sh;
}

template <typename T>
__global__ void k_bwd_pre(const Problem p) {
  const int64_t w = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= p.rows_q * p.N1) return;
  const int64_t r = w / p.N1;
  const int h = int(w % p.N1);
  const T *dO = static_cast<const T *>(p.dout) + qstore_off(p, p.do_sb, p.do_sh, p.do_st, r, h);
  const T *O = static_cast<const T *>(p.out) + qstore_off(p, p.o_sb, p.o_sh, p.o_st, r, h);
  float acc = 0.f;
  for (int d = lane * 2; d < p.D; d += 64) {
    const float2 a = MmaOp<T>::unpack(*reinterpret_cast<const uint32_t *>(dO + d));
    const float2 c = MmaOp<T>::unpack(*reinterpret_cast<const uint32_t *>(O + d));
    acc = fmaf(a.x, c.x, fmaf(a.y, c.y, acc));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) p.dsum[r * p.N1 + h] = acc;
}

struct StepCursor {
  int hh;  // q head within the group
  int e;   // entry of that head's inverted list
  int st;  // 64-row step inside the query block
};

template <int D, typename T>
__global__ void __launch_bounds__(kBwdThreads, 1) k_bwd_main(const Problem p) {
  using Op = MmaOp<T>;
  constexpr int BN = kBwdBN, BM = kBwdBM, CH = D / 8;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  T *sK = reinterpret_cast<T *>(smem_raw);
  T *sV = sK + BN * D;
  T *sQ = sV + BN * D;         // [2][BM][D]
  T *sdO = sQ + 2 * BM * D;    // [2][BM][D]
  T *sdS = sdO + 2 * BM * D;   // [BN][BM]  (dS^T)
  float *sL = reinterpret_cast<float *>(sdS + BN * BM);  // [2][BM] lse * log2(e)
  float *sDs = sL + 2 * BM;                              // [2][BM] Dsum
  __shared__ int s_item;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int n_items = int(p.status[kStBwdItems]);
  const int TK = int(p.status[kStTK]);
  const float kLog2e = 1.4426950408889634f;
  const int steps_per_block = p.BQ / BM;
  const T *qg = static_cast<const T *>(p.q);
  const T *kg = static_cast<const T *>(p.k);
  const T *vg = static_cast<const T *>(p.v);
  const T *dog = static_cast<const T *>(p.dout);

  for (;;) {
    if (tid == 0) s_item = int(atomicAdd(p.status + kStBwdNext, 1u));
    __syncthreads();
    const int it = s_item;
    if (it >= n_items) break;
    const int id = p.bwd_items[it];
    const int ks = id % p.ksl;
    const int gk = (id / p.ksl) % TK;
    const int h2 = id / (p.ksl * TK);
    const int b = p.kb_batch[gk];
    const BatchInfo bi = p.batch[b];
    const int j = gk - bi.koff;
    const int u0 = j * p.BKV + ks * BN;
    const int kvlen = bi.kvlen;
    const int wb = min(BN, bi.kvst - u0);  // rows of this item that exist in storage
    const int pg = p.kv_layout == BSA_LAYOUT_PA_BBND ? kv_page(p, b, u0) : 0;
    if (pg < 0) {
      if (tid == 0) atomicOr(p.status + kStFlags, BSA_FLAG_BAD_PAGE);
      __syncthreads();
      continue;
    }

    // ---- K, V chunk -> shared (rows past kvlen are zero)
    for (int c = tid; c < BN * CH; c += kBwdThreads) {
      const int r = c / CH, ch = c % CH;
      const bool ok = u0 + r < kvlen;
      const int u = ok ? u0 + r : u0;
      cp_async16(smem_u32(sK + swz<D>(r, ch * 8)),
                 kg + kv_row(p, p.k_sb, p.k_sh, p.k_st, bi, b, h2, u, pg) + ch * 8, ok ? 16 : 0);
      cp_async16(smem_u32(sV + swz<D>(r, ch * 8)),
                 vg + kv_row(p, p.v_sb, p.v_sh, p.v_st, bi, b, h2, u, pg) + ch * 8, ok ? 16 : 0);
    }

    // ---- step cursor over (group head, inverted-list entry, 64-row step)
    auto list_lo = [&](int hh) {
      const int h1 = h2 * p.g + hh;
      const int hi = p.Hidx == p.N1 ? h1 : h2;
      return int64_t(hi) * TK + gk;
    };
    auto settle = [&](StepCursor c) {
      while (c.hh < p.g) {
        const int64_t li = list_lo(c.hh);
        const int len = p.inv_off[li + 1] - p.inv_off[li];
        if (c.e < len) {
          const int i = p.inv_list[p.inv_off[li] + c.e];
          if (c.st < steps_per_block && i * p.BQ + c.st * BM < bi.qlen) return c;
          ++c.e;
          c.st = 0;
          continue;
        }
        ++c.hh;
        c.e = 0;
        c.st = 0;
      }
      return c;
    };
    auto q_start = [&](const StepCursor &c) {
      return p.inv_list[p.inv_off[list_lo(c.hh)] + c.e] * p.BQ + c.st * BM;
    };
    auto load_step = [&](int buf, const StepCursor &c) {
      const int h1 = h2 * p.g + c.hh;
      const int t0 = q_start(c);
      T *dq_ = sQ + buf * BM * D;
      T *ddo = sdO + buf * BM * D;
      for (int x = tid; x < BM * CH; x += kBwdThreads) {
        const int r = x / CH, ch = x % CH;
        const bool ok = t0 + r < bi.qlen;
        const int t = ok ? t0 + r : t0;
        cp_async16(smem_u32(dq_ + swz<D>(r, ch * 8)),
                   qg + q_row(p.q_sb, p.q_sh, p.q_st, bi, b, h1, t) + ch * 8, ok ? 16 : 0);
        cp_async16(smem_u32(ddo + swz<D>(r, ch * 8)),
                   dog + q_row(p.do_sb, p.do_sh, p.do_st, bi, b, h1, t) + ch * 8, ok ? 16 : 0);
      }
      if (tid < BM) {
        const bool ok = t0 + tid < bi.qlen;
        float lv = INFINITY, dv = 0.f;
        if (ok) {
          lv = p.lse[q_row(p.l_sb, p.l_sh, p.l_st, bi, b, h1, t0 + tid)] * kLog2e;
          if (!(lv > -INFINITY)) lv = INFINITY;  // no selected key: P = 0
          const int64_t srow = p.q_layout == BSA_LAYOUT_BNSD ? int64_t(b) * p.Sq + t0 + tid
                                                             : bi.q_tok0 + t0 + tid;
          dv = p.dsum[srow * p.N1 + h1];
        }
        sL[buf * BM + tid] = lv;
        sDs[buf * BM + tid] = dv;
      }
    };

    StepCursor cur = settle(StepCursor{0, 0, 0});
    if (cur.hh < p.g) load_step(0, cur);
    cp_async_commit();

    float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
    for (int d = 0; d < D / 8; ++d) {
      dk[d][0] = dk[d][1] = dk[d][2] = dk[d][3] = 0.f;
      dv[d][0] = dv[d][1] = dv[d][2] = dv[d][3] = 0.f;
    }
    const int kr0 = warp * 16 + g8, kr1 = kr0 + 8;  // this thread's kv rows
    const bool kv_ok0 = u0 + kr0 < kvlen, kv_ok1 = u0 + kr1 < kvlen;
    int buf = 0;

    while (cur.hh < p.g) {
      StepCursor nxt = cur;
      ++nxt.st;
      nxt = settle(nxt);
      if (nxt.hh < p.g) load_step(buf ^ 1, nxt);
      cp_async_commit();
      cp_async_wait<1>();
      __syncthreads();
      const T *Qt = sQ + buf * BM * D;
      const T *dOt = sdO + buf * BM * D;
      const float *Lt = sL + buf * BM;
      const float *Dt = sDs + buf * BM;
      const int h1 = h2 * p.g + cur.hh;
      const int t0 = q_start(cur);

      // S^T = K Q^T : 16 kv rows x 64 q columns per warp
      float s[BM / 8][4];
#pragma unroll
      for (int n = 0; n < BM / 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a[4];
        ldsm_x4(smem_u32(sK + swz<D>(warp * 16 + (lane & 15), kk * 16 + (lane >> 4) * 8)), a[0],
                a[1], a[2], a[3]);
#pragma unroll
        for (int np = 0; np < BM / 16; ++np) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(smem_u32(Qt + swz<D>(np * 16 + (lane & 7) + ((lane >> 4) << 3),
                                       kk * 16 + ((lane >> 3) & 1) * 8)),
                  b0, b1, b2, b3);
          Op::run(s[2 * np], a, b0, b1);
          Op::run(s[2 * np + 1], a, b2, b3);
        }
      }
      // P^T = exp(scale*S^T - lse), zero for kv rows past kvlen / padded q rows
#pragma unroll
      for (int n = 0; n < BM / 8; ++n) {
        const int c = n * 8 + 2 * t4;
        const float l0 = Lt[c], l1 = Lt[c + 1];
        s[n][0] = kv_ok0 ? ex2(fmaf(s[n][0], p.scale_log2, -l0)) : 0.f;
        s[n][1] = kv_ok0 ? ex2(fmaf(s[n][1], p.scale_log2, -l1)) : 0.f;
        s[n][2] = kv_ok1 ? ex2(fmaf(s[n][2], p.scale_log2, -l0)) : 0.f;
        s[n][3] = kv_ok1 ? ex2(fmaf(s[n][3], p.scale_log2, -l1)) : 0.f;
      }
      // dP^T = V dOut^T
      float dp[BM / 8][4];
#pragma unroll
      for (int n = 0; n < BM / 8; ++n) dp[n][0] = dp[n][1] = dp[n][2] = dp[n][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a[4];
        ldsm_x4(smem_u32(sV + swz<D>(warp * 16 + (lane & 15), kk * 16 + (lane >> 4) * 8)), a[0],
                a[1], a[2], a[3]);
#pragma unroll
        for (int np = 0; np < BM / 16; ++np) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(smem_u32(dOt + swz<D>(np * 16 + (lane & 7) + ((lane >> 4) << 3),
                                        kk * 16 + ((lane >> 3) & 1) * 8)),
                  b0, b1, b2, b3);
          Op::run(dp[2 * np], a, b0, b1);
          Op::run(dp[2 * np + 1], a, b2, b3);
        }
      }
      // dS^T = P^T o (dP^T - Dsum); both rounded to the input dtype as MMA operands
      uint32_t pa[BM / 16][4], da[BM / 16][4];
#pragma unroll
      for (int n = 0; n < BM / 8; ++n) {
        const int c = n * 8 + 2 * t4;
        const float d0 = Dt[c], d1 = Dt[c + 1];
        dp[n][0] = s[n][0] * (dp[n][0] - d0);
        dp[n][1] = s[n][1] * (dp[n][1] - d1);
        dp[n][2] = s[n][2] * (dp[n][2] - d0);
        dp[n][3] = s[n][3] * (dp[n][3] - d1);
      }
#pragma unroll
      for (int kk = 0; kk < BM / 16; ++kk) {
        pa[kk][0] = Op::pack(s[2 * kk][0], s[2 * kk][1]);
        pa[kk][1] = Op::pack(s[2 * kk][2], s[2 * kk][3]);
        pa[kk][2] = Op::pack(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        pa[kk][3] = Op::pack(s[2 * kk + 1][2], s[2 * kk + 1][3]);
        da[kk][0] = Op::pack(dp[2 * kk][0], dp[2 * kk][1]);
        da[kk][1] = Op::pack(dp[2 * kk][2], dp[2 * kk][3]);
        da[kk][2] = Op::pack(dp[2 * kk + 1][0], dp[2 * kk + 1][1]);
        da[kk][3] = Op::pack(dp[2 * kk + 1][2], dp[2 * kk + 1][3]);
      }
      // stash dS^T for the dQ product: sdS[kv row][q col]
#pragma unroll
      for (int kk = 0; kk < BM / 16; ++kk) {
        *reinterpret_cast<uint32_t *>(sdS + swz<BM>(kr0, kk * 16 + 2 * t4)) = da[kk][0];
        *reinterpret_cast<uint32_t *>(sdS + swz<BM>(kr1, kk * 16 + 2 * t4)) = da[kk][1];
        *reinterpret_cast<uint32_t *>(sdS + swz<BM>(kr0, kk * 16 + 8 + 2 * t4)) = da[kk][2];
        *reinterpret_cast<uint32_t *>(sdS + swz<BM>(kr1, kk * 16 + 8 + 2 * t4)) = da[kk][3];
      }
      // dV += P^T dOut ; dK += dS^T Q
#pragma unroll
      for (int kk = 0; kk < BM / 16; ++kk) {
#pragma unroll
        for (int dpi = 0; dpi < D / 16; ++dpi) {
          const int r = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int c = dpi * 16 + (lane >> 4) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(smem_u32(dOt + swz<D>(r, c)), b0, b1, b2, b3);
          Op::run(dv[2 * dpi], pa[kk], b0, b1);
          Op::run(dv[2 * dpi + 1], pa[kk], b2, b3);
          ldsm_x4_t(smem_u32(Qt + swz<D>(r, c)), b0, b1, b2, b3);
          Op::run(dk[2 * dpi], da[kk], b0, b1);
          Op::run(dk[2 * dpi + 1], da[kk], b2, b3);
        }
      }
      __syncthreads();  // every warp's dS^T is in shared memory

      // dQacc[q rows] += dS K : warp -> 16 q rows x D/2 columns
      {
        const int qr = (warp & 3) * 16;
        const int dc = (warp >> 2) * (D / 2);
        float acc[D / 16][4];
#pragma unroll
        for (int n = 0; n < D / 16; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          uint32_t a[4];
          ldsm_x4_t(smem_u32(sdS + swz<BM>(kk * 16 + (lane & 7) + ((lane >> 4) << 3),
                                           qr + ((lane >> 3) & 1) * 8)),
                    a[0], a[1], a[2], a[3]);
#pragma unroll
          for (int np = 0; np < D / 32; ++np) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(smem_u32(sK + swz<D>(kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8,
                                           dc + np * 16 + (lane >> 4) * 8)),
                      b0, b1, b2, b3);
            Op::run(acc[2 * np], a, b0, b1);
            Op::run(acc[2 * np + 1], a, b2, b3);
          }
        }
        const int q0 = qr + g8, q1 = q0 + 8;
        const int64_t base_row = p.q_layout == BSA_LAYOUT_BNSD ? int64_t(b) * p.Sq : bi.q_tok0;
        float *dqa = p.dq_acc + int64_t(h1) * D;
#pragma unroll
        for (int n = 0; n < D / 16; ++n) {
          const int d = dc + n * 8 + 2 * t4;
          if (t0 + q0 < bi.qlen)
            atomicAdd(reinterpret_cast<float2 *>(dqa + (base_row + t0 + q0) * p.N1 * D + d),
                      make_float2(acc[n][0], acc[n][1]));
          if (t0 + q1 < bi.qlen)
            atomicAdd(reinterpret_cast<float2 *>(dqa + (base_row + t0 + q1) * p.N1 * D + d),
                      make_float2(acc[n][2], acc[n][3]));
        }
      }
      __syncthreads();
      cur = nxt;
      buf ^= 1;
    }
    cp_async_wait<0>();
    __syncthreads();

    // ---- epilogue: dK *= scale, stage through shared, coalesced stores
#pragma unroll
    for (int d = 0; d < D / 8; ++d) {
      *reinterpret_cast<uint32_t *>(sK + swz<D>(kr0, d * 8 + 2 * t4)) =
          Op::pack(dk[d][0] * p.scale, dk[d][1] * p.scale);
      *reinterpret_cast<uint32_t *>(sK + swz<D>(kr1, d * 8 + 2 * t4)) =
          Op::pack(dk[d][2] * p.scale, dk[d][3] * p.scale);
      *reinterpret_cast<uint32_t *>(sV + swz<D>(kr0, d * 8 + 2 * t4)) = Op::pack(dv[d][0], dv[d][1]);
      *reinterpret_cast<uint32_t *>(sV + swz<D>(kr1, d * 8 + 2 * t4)) = Op::pack(dv[d][2], dv[d][3]);
    }
    __syncthreads();
    T *dkg = static_cast<T *>(p.dk);
    T *dvg = static_cast<T *>(p.dv);
    for (int c = tid; c < BN * CH; c += kBwdThreads) {
      const int r = c / CH, ch = c % CH;
      if (r < wb) {
        const int u = u0 + r;
        *reinterpret_cast<uint4 *>(dkg + kv_row(p, p.dk_sb, p.dk_sh, p.dk_st, bi, b, h2, u, pg) +
                                   ch * 8) = *reinterpret_cast<const uint4 *>(sK + swz<D>(r, ch * 8));
        *reinterpret_cast<uint4 *>(dvg + kv_row(p, p.dv_sb, p.dv_sh, p.dv_st, bi, b, h2, u, pg) +
                                   ch * 8) = *reinterpret_cast<const uint4 *>(sV + swz<D>(r, ch * 8));
      }
    }
    __syncthreads();
  }
}

// dq = dtype(scale * dQacc) for every q storage row
template <typename T>
__global__ void k_dq_convert(const Problem p) {
  const int64_t n8 = p.rows_q * p.N1 * (p.D / 8);
  const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= n8) return;
  const int64_t e = idx * 8;
  const int d = int(e % p.D);
  const int h = int((e / p.D) % p.N1);
  const int64_t r = e / (int64_t(p.D) * p.N1);
  const float4 x0 = *reinterpret_cast<const float4 *>(p.dq_acc + e);
  const float4 x1 = *reinterpret_cast<const float4 *>(p.dq_acc + e + 4);
  uint4 o;
  o.x = MmaOp<T>::pack(x0.x * p.scale, x0.y * p.scale);
  o.y = MmaOp<T>::pack(x0.z * p.scale, x0.w * p.scale);
  o.z = MmaOp<T>::pack(x1.x * p.scale, x1.y * p.scale);
  o.w = MmaOp<T>::pack(x1.z * p.scale, x1.w * p.scale);
  *reinterpret_cast<uint4 *>(static_cast<T *>(p.dq) + qstore_off(p, p.dq_sb, p.dq_sh, p.dq_st, r, h) +
                             d) = o;
}

// zeros for the kv rows of each batch that no backward item covers:
// [round_up(kvlen, 128), kvst) -- stored rows past the used length
template <typename T>
__global__ void k_kv_zero_tail(const Problem p) {
  const int b = blockIdx.y;
  const BatchInfo bi = p.batch[b];
  const int lo = ((bi.kvlen + kSlice - 1) / kSlice) * kSlice;
  const int64_t rows = bi.kvst > lo ? bi.kvst - lo : 0;
  const int CH = p.D / 8;
  const int64_t total = rows * p.N2 * CH;
  T *dkg = static_cast<T *>(p.dk);
  T *dvg = static_cast<T *>(p.dv);
  for (int64_t x = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; x < total;
       x += int64_t(gridDim.x) * blockDim.x) {
    const int ch = int(x % CH);
    const int h2 = int((x / CH) % p.N2);
    const int u = lo + int(x / (int64_t(CH) * p.N2));
    int pg = 0;
    if (p.kv_layout == BSA_LAYOUT_PA_BBND) {
      pg = kv_page(p, b, u);
      if (pg < 0) continue;
    }
    const uint4 z = make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4 *>(dkg + kv_row(p, p.dk_sb, p.dk_sh, p.dk_st, bi, b, h2, u, pg) + ch * 8) = z;
    *reinterpret_cast<uint4 *>(dvg + kv_row(p, p.dv_sb, p.dv_sh, p.dv_st, bi, b, h2, u, pg) + ch * 8) = z;
  }
}

template <int D, typename T>
cudaError_t launch_bwd_t(const Problem &p, cudaStream_t s) {
  const int smem = (2 * kBwdBN * D + 4 * kBwdBM * D + kBwdBN * kBwdBM) * int(sizeof(T)) +
                   4 * kBwdBM * int(sizeof(float));
  cudaError_t e = cudaFuncSetAttribute(k_bwd_main<D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = p.bwd_slots < num_sms() ? p.bwd_slots : num_sms();
  if (grid <= 0) return cudaSuccess;
  k_bwd_main<D, T><<<unsigned(grid), kBwdThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_pre(const Problem &p, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(p.dq_acc, 0, size_t(p.rows_q) * p.N1 * p.D * sizeof(float), s);
  if (e != cudaSuccess) return e;
  const int64_t warps = p.rows_q * p.N1;
  const unsigned grid = unsigned((warps * 32 + 255) / 256);
  if (p.dtype == BSA_BF16) k_bwd_pre<__nv_bfloat16><<<grid, 256, 0, s>>>(p);
  else k_bwd_pre<__half><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_bwd_main(const Problem &p, cudaStream_t s) {
  if (p.dtype == BSA_BF16)
    return p.D == 64 ? launch_bwd_t<64, __nv_bfloat16>(p, s) : launch_bwd_t<128, __nv_bfloat16>(p, s);
  return p.D == 64 ? launch_bwd_t<64, __half>(p, s) : launch_bwd_t<128, __half>(p, s);
}

cudaError_t launch_bwd_post(const Problem &p, cudaStream_t s) {
  const int64_t n8 = p.rows_q * p.N1 * (p.D / 8);
  const unsigned grid = unsigned((n8 + 255) / 256);
  const dim3 zgrid(64, unsigned(p.B));
  if (p.dtype == BSA_BF16) {
    k_dq_convert<__nv_bfloat16><<<grid, 256, 0, s>>>(p);
    k_kv_zero_tail<__nv_bfloat16><<<zgrid, 256, 0, s>>>(p);
  } else {
    k_dq_convert<__half><<<grid, 256, 0, s>>>(p);
    k_kv_zero_tail<__half><<<zgrid, 256, 0, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace bsa
