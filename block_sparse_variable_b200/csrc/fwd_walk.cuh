// fwd_walk.cuh -- the chunk walk of a forward work item, shared by the
// kernels that iterate query tiles over their selected kv chunks (the
// forward and the q-major dQ pass of the deterministic backward).
//
// An item is 128 query rows (sub-tile qs of global query-block row gq) of
// query head h1; it walks the compacted index row of (index head, gq) in
// order, each kept block in 128-row kv chunks that start below kvlen and,
// paged, whose page is valid.
#pragma once

#include "addr.cuh"
#include "bsa_internal.h"

namespace bsa {
namespace {

struct Chunk {
  int x, c;  // compacted-row position, 128-row chunk of that kv block
};

// every role walks the same chunk sequence of an item.  Packed heads
// (p.pack_g > 1): tile row r is query row t0 + r % (128 / pack_g) of head
// h1 + r / (128 / pack_g); rows counts the valid rows of each head.
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
// The same walk for a role on the critical path: the current kv block id is
// held in a register and the next one is loaded a block ahead, so that no
// load of the index row sits between two chunks (the index is re-read
// after every memory-clobbering barrier or TMEM operation otherwise).
struct Cursor {
  int x, c, blk, nblk;  // row position, chunk of the block, block ids at x and x + 1
};
__device__ __forceinline__ int cur_u0(const ItemView &v, const Cursor &k) {
  return k.blk * v.BKV + k.c * 128;
}
__device__ __forceinline__ void cur_step(const ItemView &v, Cursor &k) {
  ++k.c;
  if (k.c >= v.ksl || cur_u0(v, k) >= v.kvlen) {
    ++k.x;
    k.c = 0;
    k.blk = k.nblk;
    k.nblk = k.x + 1 < v.ncnt ? int(v.crow[k.x + 1]) : 0;
  }
}
__device__ __forceinline__ void cur_settle(const Problem &p, const ItemView &v, Cursor &k) {
  if (p.kv_layout != BSA_LAYOUT_PA_BBND) return;
  int pg;
  while (k.x < v.ncnt && !page_ok(p, v, cur_u0(v, k), pg)) cur_step(v, k);
}
__device__ __forceinline__ Cursor cur_begin(const Problem &p, const ItemView &v) {
  Cursor k{0, 0, v.ncnt > 0 ? int(v.crow[0]) : 0, v.ncnt > 1 ? int(v.crow[1]) : 0};
  cur_settle(p, v, k);
  return k;
}
__device__ __forceinline__ void cur_next(const Problem &p, const ItemView &v, Cursor &k) {
  cur_step(v, k);
  cur_settle(p, v, k);
}

// The chunk count of an item, by a whole (converged) warp: each lane takes
// index entries lane, lane + 32, ... so their loads are in flight together,
// then the counts are summed.
__device__ __forceinline__ int count_chunks_warp(const Problem &p, const ItemView &v, int lane) {
  int n = 0;
  for (int x = lane; x < v.ncnt; x += 32) {
    const int base = int(v.crow[x]) * v.BKV;
    for (int c = 0; c < v.ksl; ++c) {
      const int u0 = base + c * 128;
      if (u0 >= v.kvlen) break;
      int pg;
      if (page_ok(p, v, u0, pg)) ++n;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
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

// a packed-head item (p.pack_g > 1): rows [t0, t0 + 128/g) of the query
// block for heads h1 .. h1 + g - 1 of kv head h2 (whose index row they share)
__device__ __forceinline__ ItemView item_view_packed(const Problem &p, int id) {
  ItemView v;
  const int qs = id % p.fsub;
  const int gq = (id / p.fsub) % p.Rg;
  v.h2 = id / (p.fsub * p.Rg);
  v.h1 = v.h2 * p.g;
  v.b = p.row_batch[gq];
  v.bi = p.batch[v.b];
  const int i = gq - v.bi.qoff;
  const int R = 128 / p.pack_g;
  v.t0 = i * p.BQ + qs * R;
  v.rows = min(R, v.bi.qlen - v.t0);
  const int64_t ci = int64_t(v.h2) * p.Rg + gq;  // Hidx == N2
  v.crow = p.comp + ci * p.W;
  v.ncnt = p.ncomp[ci];
  v.kvlen = v.bi.kvlen;
  v.ksl = p.ksl;
  v.BKV = p.BKV;
  return v;
}

}  // namespace
}  // namespace bsa
