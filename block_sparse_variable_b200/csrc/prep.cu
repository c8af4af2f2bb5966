// prep.cu -- on-device builders that run before the attention kernels:
//   * batch geometry from cu_seqlens / seqused_kv (lengths, block counts,
//     packed-row offsets, row -> batch maps);
//   * index compaction: drop 0xFFFF and invalid entries of every index row
//     (BlitzSparseAttention "sabi": ascending ids, 0xFFFF = unused slot) and
//     count the forward work of each (head, 128-row query slice);
//   * the KV-major inverse of the index (GenericBlockSparseAttention,
//     layoutSparsePattern 5/7: the query blocks that chose each kv block),
//     as CSR, plus the backward work of each (kv head, 128-row kv slice);
//   * the load-balanced work lists: item ids sorted by cost descending then
//     id ascending (longest first, ties head-major), by a per-CTA bitonic
//     sort of chunks of up to 4096 keys followed by a merge by rank.
#include <cuda_runtime.h>

#include <cmath>

#include "bsa_internal.h"
#include "launch.cuh"

namespace bsa {
namespace {

__device__ __forceinline__ int64_t cdiv64(int64_t a, int64_t b) { return (a + b - 1) / b; }

__global__ void k_geometry(Problem p) {
  griddep_wait();
  griddep_launch_next();
  __shared__ uint32_t sflags;
  __shared__ int64_t s_sum_nq;
  uint32_t *st = p.status;
  for (int i = threadIdx.x; i < kStWords; i += blockDim.x) st[i] = 0;
  for (int64_t r = threadIdx.x; r < p.Rg; r += blockDim.x) p.row_batch[r] = -1;
  for (int64_t r = threadIdx.x; r < p.tk_max; r += blockDim.x) p.kb_batch[r] = -1;
  if (threadIdx.x == 0) sflags = 0;
  __syncthreads();

  for (int b = threadIdx.x; b < p.B; b += blockDim.x) {
    uint32_t f = 0;
    int64_t qlen = p.Sq, q0 = 0, kvst = 0, kv0 = 0;
    if (p.q_layout == BSA_LAYOUT_TND) {
      const int64_t a = p.cu_q[b], e = p.cu_q[b + 1];
      if (a < 0 || e < a || e > p.Tq) { f |= BSA_FLAG_BAD_SEQLEN; qlen = 0; }
      else { qlen = e - a; q0 = a; }
    }
    if (p.kv_layout == BSA_LAYOUT_BNSD) {
      kvst = p.Skv;
    } else if (p.kv_layout == BSA_LAYOUT_PA_BBND) {
      kvst = int64_t(p.max_pages) * p.page_size;
    } else {
      const int64_t a = p.cu_kv[b], e = p.cu_kv[b + 1];
      if (a < 0 || e < a || e > p.Tkv) { f |= BSA_FLAG_BAD_SEQLEN; kvst = 0; }
      else { kvst = e - a; kv0 = a; }
    }
    int64_t kvlen = kvst;
    if (p.seqused_kv) {
      const int64_t u = p.seqused_kv[b];
      if (u < 0 || u > kvst) { f |= BSA_FLAG_BAD_SEQLEN; kvlen = 0; }
      else kvlen = u;
    }
    if (p.kv_layout == BSA_LAYOUT_PA_BBND) {
      // every table entry that covers a used kv token must name a page; the
      // tokens of a bad entry take no part (whether or not a row selects them)
      const int64_t used = cdiv64(kvlen, p.page_size);
      for (int64_t x = 0; x < used; ++x) {
        const int32_t pg = p.block_table[int64_t(b) * p.bt_s0 + x];
        if (pg < 0 || pg >= p.num_pages) f |= BSA_FLAG_BAD_PAGE;
      }
    }
    BatchInfo bi;
    bi.qlen = int32_t(qlen);
    bi.kvlen = int32_t(kvlen);
    bi.nq = int32_t(cdiv64(qlen, p.BQ));
    bi.nk = int32_t(cdiv64(kvlen, p.BKV));
    bi.qoff = 0;
    bi.koff = 0;
    bi.q_tok0 = q0;
    bi.kv_tok0 = kv0;
    // rows of dk/dv the backward may write: the stored rows, or under paging
    // the rows of the pages that cover the used length
    bi.kvst = p.kv_layout == BSA_LAYOUT_PA_BBND
                  ? int32_t(cdiv64(kvlen, p.page_size) * p.page_size)
                  : int32_t(kvst);
    bi.pad = 0;
    p.batch[b] = bi;
    if (f) atomicOr(&sflags, f);
  }
  __syncthreads();

  if (threadIdx.x == 0) {
    int64_t qo = 0, ko = 0;
    uint32_t f = 0;
    for (int b = 0; b < p.B; ++b) {
      BatchInfo &bi = p.batch[b];
      if (p.q_layout == BSA_LAYOUT_TND) { bi.qoff = int32_t(qo); qo += bi.nq; }
      else { bi.qoff = b * p.R; qo += bi.nq; }
      if (ko + bi.nk > p.tk_max) {  // only inconsistent cu_seqlens_kv reach this
        f |= BSA_FLAG_BAD_SEQLEN;
        bi.nk = 0;
        bi.kvlen = 0;
      }
      bi.koff = int32_t(ko);
      ko += bi.nk;
    }
    if (p.q_layout == BSA_LAYOUT_TND && qo > p.R) f |= BSA_FLAG_BAD_INDEX;
    st[kStTK] = uint32_t(ko);
    st[kStSumNq] = uint32_t(qo);
    s_sum_nq = qo;
    if (f) atomicOr(&sflags, f);
  }
  __syncthreads();

  // Query blocks past the last index row (TND, an index with fewer rows than
  // the lengths need) select nothing: their rows get out 0 and lse -inf in
  // the forward, dq 0 in the deterministic backward (whose dq pass visits
  // work items only; the default backward converts every accumulator row).
  // (BNSD indexes every batch with R = ceil(Sq/BQ) rows, checked on the host)
  const bool fwd = p.dq == nullptr;
  if (p.q_layout == BSA_LAYOUT_TND && s_sum_nq > p.R && (fwd || p.deterministic)) {
    const int CH = p.D / 8;  // 16-byte chunks of a 16-bit row
    for (int b = 0; b < p.B; ++b) {
      const BatchInfo bi = p.batch[b];
      const int64_t i0 = p.R - bi.qoff > 0 ? p.R - bi.qoff : 0;
      const int64_t t0 = i0 * p.BQ;
      const int64_t nrow = bi.qlen > t0 ? bi.qlen - t0 : 0;
      for (int64_t x = threadIdx.x; x < nrow * p.N1 * CH; x += blockDim.x) {
        const int ch = int(x % CH);
        const int h = int((x / CH) % p.N1);
        const int t = int(t0 + x / (int64_t(CH) * p.N1));
        const uint4 z = make_uint4(0, 0, 0, 0);
        if (fwd) {
          uint16_t *o = static_cast<uint16_t *>(p.out) + int64_t(b) * p.o_sb +
                        (bi.q_tok0 + t) * p.o_st + int64_t(h) * p.o_sh;
          reinterpret_cast<uint4 *>(o)[ch] = z;
          if (ch == 0 && p.lse)
            p.lse[int64_t(b) * p.l_sb + (bi.q_tok0 + t) * p.l_st + int64_t(h) * p.l_sh] = -INFINITY;
        } else {
          uint16_t *o = static_cast<uint16_t *>(p.dq) + int64_t(b) * p.dq_sb +
                        (bi.q_tok0 + t) * p.dq_st + int64_t(h) * p.dq_sh;
          reinterpret_cast<uint4 *>(o)[ch] = z;
        }
      }
    }
  }

  for (int b = threadIdx.x; b < p.B; b += blockDim.x) {
    const BatchInfo bi = p.batch[b];
    for (int i = 0; i < bi.nq; ++i) {
      const int64_t r = int64_t(bi.qoff) + i;
      if (r < p.Rg) p.row_batch[r] = b;
    }
    for (int j = 0; j < bi.nk; ++j) p.kb_batch[bi.koff + j] = b;
  }
  __syncthreads();
  if (threadIdx.x == 0) st[kStFlags] = sflags;
}

__device__ __forceinline__ uint64_t make_key(int32_t cost, int64_t id) {
  return (uint64_t(0xFFFFFFFFu - uint32_t(cost)) << 32) | uint64_t(uint32_t(id));
}

// one thread per (index head, global q-block row)
__global__ void k_compact(Problem p, int fwd_keys) {
  griddep_wait();
  griddep_launch_next();
  const int64_t r = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r >= int64_t(p.Hidx) * p.Rg) return;
  const int hi = int(r / p.Rg);
  const int gq = int(r % p.Rg);
  uint16_t *dst = p.comp + r * p.W;
  const int b = p.row_batch[gq];
  int n = 0, cost = 0, i = 0, qlen = 0;
  if (b >= 0) {
    const BatchInfo bi = p.batch[b];
    i = gq - bi.qoff;
    qlen = bi.qlen;
    const uint16_t *row = p.q_layout == BSA_LAYOUT_BNSD
                              ? p.index + b * p.ix_s0 + hi * p.ix_s1 + i * p.ix_s2
                              : p.index + hi * p.ix_s0 + int64_t(gq) * p.ix_s1;
    int last = -1;
    bool bad = false;
    for (int w = 0; w < p.W; ++w) {
      const int e = row[w];
      if (e == kNoBlock) continue;
      if (e >= bi.nk || e <= last) { bad = true; continue; }
      dst[n++] = uint16_t(e);
      last = e;
      const int rem = bi.kvlen - e * p.BKV;  // > 0 because e < nk
      cost += min(p.ksl, (rem + kSlice - 1) / kSlice);
    }
    if (bad) atomicOr(p.status + kStFlags, BSA_FLAG_BAD_INDEX);
  }
  for (int w = n; w < p.W; ++w) dst[w] = kNoBlock;
  p.ncomp[r] = n;
  if (!fwd_keys) return;
  int made = 0;
  if (p.pack_g > 1) {
    // packed heads (Hidx == N2, hi = h2): slot (h2*Rg + gq)*fsub + s covers
    // rows [s*R, s*R + R) of the query block for all g heads, R = 128/g
    const int R = kSlice / p.pack_g;
    for (int s = 0; s < p.fsub; ++s) {
      const int64_t slot = (int64_t(hi) * p.Rg + gq) * p.fsub + s;
      const bool exists = b >= 0 && i * p.BQ + s * R < qlen;
      p.keys[slot] = exists ? make_key(cost, slot) : kAbsentKey;
      made += exists;
    }
  } else {
    const int h_lo = p.Hidx == p.N1 ? hi : hi * p.g;
    const int h_hi = p.Hidx == p.N1 ? hi + 1 : h_lo + p.g;
    for (int h1 = h_lo; h1 < h_hi; ++h1)
      for (int qs = 0; qs < p.nsub; ++qs) {
        const int64_t slot = (int64_t(h1) * p.Rg + gq) * p.nsub + qs;
        const bool exists = b >= 0 && i * p.BQ + qs * kSlice < qlen;
        p.keys[slot] = exists ? make_key(cost, slot) : kAbsentKey;
        made += exists;
      }
  }
  if (made) atomicAdd(p.status + kStFwdItems, uint32_t(made));
}

__device__ __forceinline__ bool row_has(const uint16_t *row, int n, int j) {
  int lo = 0, hi = n;  // ascending row: binary search
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (int(row[mid]) < j) lo = mid + 1;
    else hi = mid;
  }
  return lo < n && int(row[lo]) == j;
}

// one warp per (index head, kv block) list: lane l tests query blocks l,
// l + 32, ... of the kv block's batch (binary search in the compacted row);
// mode 0 counts the blocks and their 128-row query slices, mode 1 writes the
// ascending list (ballots give each hit its place)
__global__ void k_inverse(Problem p, int mode) {
  griddep_wait();
  griddep_launch_next();
  const int64_t idx = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (idx >= int64_t(p.Hidx) * p.tk_max) return;
  const int hi = int(idx / p.tk_max);
  const int gk = int(idx % p.tk_max);
  const int TK = int(p.status[kStTK]);
  if (gk >= TK) return;
  const int b = p.kb_batch[gk];
  const int64_t li = int64_t(hi) * TK + gk;
  int cnt = 0, sub = 0;
  int pos = mode ? p.inv_off[li] : 0;
  if (b >= 0) {
    const BatchInfo bi = p.batch[b];
    const int j = gk - bi.koff;
    for (int i0 = 0; i0 < bi.nq; i0 += 32) {
      const int i = i0 + lane;
      const int64_t gq = int64_t(bi.qoff) + i;
      bool hit = false;
      if (i < bi.nq && gq < p.Rg) {
        const int64_t rr = int64_t(hi) * p.Rg + gq;
        hit = row_has(p.comp + rr * p.W, p.ncomp[rr], j);
      }
      const uint32_t m = __ballot_sync(0xffffffffu, hit);
      if (hit) {
        if (mode) p.inv_list[pos + __popc(m & ((1u << lane) - 1u))] = i;
        sub += min(p.nsub, (bi.qlen - i * p.BQ + kSlice - 1) / kSlice);
      }
      pos += __popc(m);
      cnt += __popc(m);
    }
  }
  if (!mode) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sub += __shfl_xor_sync(0xffffffffu, sub, o);
    if (lane == 0) {
      p.inv_cnt[li] = cnt;
      p.inv_sub[li] = sub;
    }
  }
}

// single CTA exclusive scan of inv_cnt[0 .. Hidx*TK) into inv_off; also the
// total of inv_sub (the backward work lists' grouping threshold)
__global__ void k_scan_offsets(Problem p) {
  griddep_wait();
  griddep_launch_next();
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry;
  __shared__ unsigned long long sub_total;
  const int64_t n = int64_t(p.Hidx) * p.status[kStTK];
  if (threadIdx.x == 0) {
    carry = 0;
    sub_total = 0;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  unsigned long long my_sub = 0;
  for (int64_t base = 0; base < n; base += blockDim.x) {
    const int64_t i = base + threadIdx.x;
    const int32_t x = i < n ? p.inv_cnt[i] : 0;
    if (i < n) my_sub += uint32_t(p.inv_sub[i]);
    int32_t s = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane == 31) warp_sums[wid] = s;
    __syncthreads();
    if (wid == 0) {
      int32_t w = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      if (lane < nw) warp_sums[lane] = w;
    }
    __syncthreads();
    const int32_t before = carry + (wid ? warp_sums[wid - 1] : 0) + s - x;
    if (i < n) p.inv_off[i] = before;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = before + x;
    __syncthreads();
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) my_sub += __shfl_xor_sync(0xffffffffu, my_sub, o);
  if (lane == 0) atomicAdd(&sub_total, my_sub);
  __syncthreads();
  if (threadIdx.x == 0) {
    p.inv_off[n] = carry;
    p.status[kStNnz] = uint32_t(carry);
    p.status[kStSubSum] = uint32_t(sub_total);
    p.status[kStSubSum + 1] = uint32_t(sub_total >> 32);
  }
}

// Backward sort key.  Items whose cost exceeds 1/512 of the list's total
// (about 0.3 of a CTA's share on a 148-SM part) come first, longest first;
// the rest follow kv head by kv head, longest first within a head, so that
// the items in flight at any time share one kv head's Q, dOut and dQ rows
// in L2.  (More than 1024 kv heads: longest first throughout.)
__device__ __forceinline__ uint64_t bwd_key(int32_t cost, int h2, int64_t id, int64_t big) {
  if (int64_t(cost) > big)
    return (uint64_t(0x7FFFFFFFu - uint32_t(cost)) << 32) | uint64_t(uint32_t(id));
  return (uint64_t(1) << 63) | (uint64_t(h2) << 53) |
         (uint64_t(0x1FFFFFu - uint32_t(min(cost, 0x1FFFFF))) << 32) | uint64_t(uint32_t(id));
}

// one thread per backward slot (h2, gk, kv slice)
__global__ void k_bwd_keys(Problem p) {
  griddep_wait();
  griddep_launch_next();
  const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= p.bwd_slots) return;
  const int TK = int(p.status[kStTK]);
  const int64_t live = int64_t(p.N2) * TK * p.ksl;
  if (idx >= live) { p.keys[idx] = kAbsentKey; return; }
  const int ks = int(idx % p.ksl);
  const int gk = int((idx / p.ksl) % TK);
  const int h2 = int(idx / (int64_t(p.ksl) * TK));
  const int b = p.kb_batch[gk];
  bool exists = false;
  int cost = 0;
  if (b >= 0) {
    const BatchInfo bi = p.batch[b];
    const int j = gk - bi.koff;
    exists = j * p.BKV + ks * kSlice < bi.kvlen;
    if (p.Hidx == p.N1) {
      for (int h1 = h2 * p.g; h1 < (h2 + 1) * p.g; ++h1) cost += p.inv_sub[int64_t(h1) * TK + gk];
    } else {
      cost = p.g * p.inv_sub[int64_t(h2) * TK + gk];
    }
  }
  // the list's total cost, counting every kv block at full length: the sum of
  // the inverse lists' query slices, times g when the group shares its lists,
  // times the kv slices per block
  const uint64_t sub = uint64_t(p.status[kStSubSum]) | (uint64_t(p.status[kStSubSum + 1]) << 32);
  const int64_t total = int64_t(sub) * (p.Hidx == p.N1 ? 1 : p.g) * p.ksl;
  const int64_t big = p.N2 <= 1024 ? total >> 9 : -1;
  p.keys[idx] = exists ? bwd_key(cost, h2, idx, big) : kAbsentKey;
  if (exists) atomicAdd(p.status + kStBwdItems, 1u);
}

__device__ __forceinline__ void cmp_swap(uint64_t &a, uint64_t &c, bool up) {
  if ((a > c) == up) { const uint64_t t = a; a = c; c = t; }
}

__device__ __forceinline__ uint64_t shfl_xor64(uint64_t x, int m) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, uint32_t(x), m);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, uint32_t(x >> 32), m);
  return (uint64_t(hi) << 32) | lo;
}

// bitonic sort (ascending) of one n-key chunk, n a power of two in
// [128, kSortChunk], by n/4 threads; thread t holds keys 4t..4t+3 in
// registers.  Stages whose partner distance j is 1 or 2 stay in the thread,
// 4 <= j <= 64 cross lanes of one warp (shuffles), j >= 128 go through shared
// memory, where consecutive such stages run in place.
// A single chunk is the whole list: its sorted keys go straight to the item
// list (`items`, else null), each real key's place being its rank.
__global__ void __launch_bounds__(kSortChunk / 4) k_sort_chunks(const uint64_t *keys,
                                                                uint64_t *sorted, int64_t slots,
                                                                int n, int32_t *items) {
  __shared__ uint64_t s[kSortChunk];
  griddep_wait();
  griddep_launch_next();
  const int t = threadIdx.x;
  const int64_t base = int64_t(blockIdx.x) * n;
  uint64_t v[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int64_t e = base + 4 * t + r;
    v[r] = e < slots ? keys[e] : kAbsentKey;
  }
  // a chunk already in order (equal costs: the keys ascend with the id)
  // needs no network
  {
    const uint64_t next = __shfl_down_sync(0xffffffffu, v[0], 1);
    bool in_order = v[0] <= v[1] && v[1] <= v[2] && v[2] <= v[3] &&
                    ((t & 31) == 31 || v[3] <= next);
    if ((t & 31) == 0) s[t >> 5] = v[0];  // each warp's first key, for the warp before
    __syncthreads();
    if ((t & 31) == 31 && t + 1 < int(blockDim.x)) in_order = in_order && v[3] <= s[(t >> 5) + 1];
    if (__syncthreads_and(in_order)) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        if (!items) sorted[base + 4 * t + r] = v[r];
        else if (v[r] != kAbsentKey) items[4 * t + r] = int32_t(uint32_t(v[r] & 0xFFFFFFFFu));
      }
      return;
    }
  }
  for (int k = 2; k <= n; k <<= 1) {
    int j = k >> 1;
    if (j >= 128) {
#pragma unroll
      for (int r = 0; r < 4; ++r) s[4 * t + r] = v[r];
      __syncthreads();
      for (; j >= 128; j >>= 1) {
        for (int q = t; q < (n >> 1); q += blockDim.x) {
          const int i = ((q & ~(j - 1)) << 1) | (q & (j - 1));  // bit j of i clear
          uint64_t a = s[i], c = s[i | j];
          cmp_swap(a, c, (i & k) == 0);
          s[i] = a;
          s[i | j] = c;
        }
        __syncthreads();
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) v[r] = s[4 * t + r];
      __syncthreads();
    }
    const bool up = ((4 * t) & k) == 0;  // the same for the thread's 4 keys once k >= 4
    for (; j >= 4; j >>= 1) {
      const bool keep_min = (((4 * t) & j) == 0) == up;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const uint64_t o = shfl_xor64(v[r], j >> 2);
        v[r] = keep_min ? (o < v[r] ? o : v[r]) : (o > v[r] ? o : v[r]);
      }
    }
    if (j == 2) {
      cmp_swap(v[0], v[2], up);
      cmp_swap(v[1], v[3], up);
    }
    // j == 1 (for k == 2 the direction flips between the thread's two pairs)
    cmp_swap(v[0], v[1], k == 2 ? true : up);
    cmp_swap(v[2], v[3], k == 2 ? false : up);
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    if (!items) sorted[base + 4 * t + r] = v[r];
    else if (v[r] != kAbsentKey) items[4 * t + r] = int32_t(uint32_t(v[r] & 0xFFFFFFFFu));
  }
}

// final position of every real key = its place in its chunk + the keys
// below it in every other chunk (keys are unique: the id is in the low word)
__global__ void k_rank(const uint64_t *sorted, int64_t nchunks, int n, int32_t *items) {
  griddep_wait();
  griddep_launch_next();
  const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= nchunks * n) return;
  const uint64_t key = sorted[idx];
  if (key == kAbsentKey) return;
  const int64_t c = idx / n;
  int64_t rank = idx - c * n;
  for (int64_t o = 0; o < nchunks; ++o) {
    if (o == c) continue;
    const uint64_t *a = sorted + o * n;
    int lo = 0, hi = n;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (a[mid] < key) lo = mid + 1;
      else hi = mid;
    }
    rank += lo;
  }
  items[rank] = int32_t(uint32_t(key & 0xFFFFFFFFu));
}

}  // namespace

cudaError_t launch_prep_geometry(const Problem &p, cudaStream_t s) {
  cudaError_t e = launch_dep(k_geometry, dim3(1), dim3(1024), 0, s, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_prep_compact(const Problem &p, bool fwd_keys, cudaStream_t s) {
  const int64_t n = int64_t(p.Hidx) * p.Rg;
  if (n > 0) {
    cudaError_t e = launch_dep(k_compact, dim3(unsigned((n + 255) / 256)), dim3(256), 0, s, p, fwd_keys ? 1 : 0);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

cudaError_t launch_sort_items(const Problem &p, int64_t slots_pad, int32_t *items, cudaStream_t s) {
  const bool fwd = items == p.fwd_items;
  const int64_t slots = fwd ? p.fwd_slots : p.bwd_slots;
  if (slots_pad == 0 || slots == 0) return cudaGetLastError();
  // one chunk of the next power of two (at least 128) when the slots fit in
  // one, else kSortChunk-key chunks (slots_pad is a multiple of kSortChunk)
  int n = 128;
  while (n < slots && n < kSortChunk) n <<= 1;
  const int64_t nchunks = (slots + n - 1) / n;
  cudaError_t e = launch_dep(k_sort_chunks, dim3(unsigned(nchunks)), dim3(unsigned(n / 4)), 0, s,
                             (const uint64_t *)p.keys, p.sorted, slots, n,
                             nchunks == 1 ? items : (int32_t *)nullptr);
  if (e != cudaSuccess) return e;
  if (nchunks > 1) {
    e = launch_dep(k_rank, dim3(unsigned((nchunks * n + 255) / 256)), dim3(256), 0, s,
                   (const uint64_t *)p.sorted, nchunks, n, items);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

cudaError_t launch_prep_inverse(const Problem &p, cudaStream_t s) {
  const int64_t n = int64_t(p.Hidx) * p.tk_max;  // lists, one warp each
  const unsigned grid = unsigned((n * 32 + 255) / 256);
  cudaError_t e = cudaSuccess;
  if (n > 0 && (e = launch_dep(k_inverse, dim3(grid), dim3(256), 0, s, p, 0)) != cudaSuccess) return e;
  if ((e = launch_dep(k_scan_offsets, dim3(1), dim3(1024), 0, s, p)) != cudaSuccess) return e;
  if (n > 0 && (e = launch_dep(k_inverse, dim3(grid), dim3(256), 0, s, p, 1)) != cudaSuccess) return e;
  if (p.bwd_slots > 0 &&
      (e = launch_dep(k_bwd_keys, dim3(unsigned((p.bwd_slots + 255) / 256)), dim3(256), 0, s, p)) != cudaSuccess)
    return e;
  return cudaGetLastError();
}

}  // namespace bsa
