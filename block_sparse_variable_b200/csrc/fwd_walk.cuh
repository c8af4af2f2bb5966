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

}  // namespace
}  // namespace bsa
