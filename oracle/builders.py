"""Oracle for the index builders: batch geometry, compacted index rows, the
inverted (KV-major) index and the two load-balanced work lists.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Definitions (the CUDA library must reproduce these exactly):

* Batch geometry.  qlen_b: BNSD the stored S; TND cu_q[b+1]-cu_q[b].  The
  stored kv length is S (BNSD), the cu_kv difference (TND) or
  max_pages*page (PA_BBND); kvlen_b is seqused_kv[b] when given, else the
  stored length.  A length that contradicts its storage (negative,
  decreasing cu, past the end, seqused > stored) sets BAD_SEQLEN and counts
  as 0.  nq_b = ceil(qlen_b/BQ), nk_b = ceil(kvlen_b/BKV).  Global query
  block rows: gq = qoff_b + i with qoff_b = sum_{b'<b} nq_b' (TND, the
  GenericBlockSparseAttention "totalQBlocks" packing) or b*R (BNSD);
  global kv blocks gk = koff_b + j with koff_b = sum_{b'<b} nk_b'.

* Compacted rows (BlitzSparseAttention "sabi": 0xFFFF = unused, rows
  ascending): for index head hi and global row gq, the accepted entries
  of the raw row, left-aligned, the rest 0xFFFF; an entry >= nk_b or not
  above the previous accepted one is dropped and sets BAD_INDEX.  TND rows
  that the lengths do not reach stay empty; lengths that need more rows
  than the index has set BAD_INDEX.

* Inverted index (GenericBlockSparseAttention layoutSparsePattern 5/7:
  "which Q blocks chose each KV block"): CSR over (hi, gk) in that order,
  each list the ascending batch-local q blocks i whose compacted row holds j.

* Forward work list: one item per (h1, gq, qsub) with qsub a 128-row slice
  of the q block holding at least one valid row; id = (h1*Rg + gq)*nsub +
  qsub, nsub = BQ/128; cost = number of (accepted block, 128-column slice)
  pairs whose slice starts below kvlen_b.  When the g = N1/N2 query heads of
  a group share their index row (Hidx == N2, GenericBlockSparseAttention
  isPackedGQA) and g is 2, 4, 8 or 16, the forward packs them: one item per
  (h2, gq, slice) with slice a run of R = 128/g rows of the q block holding
  at least one valid row, id = (h2*Rg + gq)*(BQ/R) + slice, covering those
  rows of all g heads; the cost is the same chunk count.  Backward work list: one item per
  (h2, gk, ksub) with the 128-row kv slice starting below kvlen_b; id =
  (h2*TK + gk)*ksubn + ksub; cost = sum over the group's q heads h1 and
  the listed q blocks i of the 128-row q slices holding a valid row.  The
  forward list: cost descending, then id ascending (longest-processing-time
  first, ties kept head-major).  The backward list: the items whose cost
  exceeds 1/512 of the list's total first, cost descending; then the rest
  kv head by kv head, cost descending within a head (bwd_worklist has the
  exact rule).  Items of cost 0 stay: they write zeros.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import List

import numpy as np
import torch

NO_BLOCK = 0xFFFF
BAD_INDEX, BAD_SEQLEN, BAD_PAGE = 1, 2, 4


def _cdiv(a, b):
    return -(-a // b)


@dataclass
class Geometry:
    qlen: List[int]
    kvlen: List[int]
    nq: List[int]
    nk: List[int]
    qoff: List[int]
    koff: List[int]
    Rg: int          # global query-block rows
    TK: int          # global kv blocks
    flags: int


def geometry(p) -> Geometry:
    fl = 0
    B = p.B
    qlen, kvlen = [], []
    for b in range(B):
        if p.layout_q == "TND":
            a, e = int(p.cu_q[b]), int(p.cu_q[b + 1])
            if a < 0 or e < a or e > p.q.shape[0]:
                fl |= BAD_SEQLEN
                qlen.append(0)
            else:
                qlen.append(e - a)
        else:
            qlen.append(int(p.q.shape[2]))
        if p.layout_kv == "BNSD":
            st = int(p.k.shape[2])
        elif p.layout_kv == "PA_BBND":
            st = int(p.block_table.shape[1]) * int(p.k.shape[1])
        else:
            a, e = int(p.cu_kv[b]), int(p.cu_kv[b + 1])
            if a < 0 or e < a or e > p.k.shape[0]:
                fl |= BAD_SEQLEN
                st = 0
            else:
                st = e - a
        if p.seqused_kv is not None:
            u = int(p.seqused_kv[b])
            if u < 0 or u > st:
                fl |= BAD_SEQLEN
                u = 0
            kvlen.append(u)
        else:
            kvlen.append(st)
    nq = [_cdiv(x, p.BQ) for x in qlen]
    nk = [_cdiv(x, p.BKV) for x in kvlen]
    R = int(p.index.shape[-2])
    if p.layout_q == "TND":
        qoff = [int(x) for x in np.concatenate([[0], np.cumsum(nq)])[:B]]
        Rg = R
        if sum(nq) > R:
            fl |= BAD_INDEX
    else:
        qoff = [b * R for b in range(B)]
        Rg = B * R
    koff = [int(x) for x in np.concatenate([[0], np.cumsum(nk)])[:B]]
    return Geometry(qlen, kvlen, nq, nk, qoff, koff, Rg, int(sum(nk)), fl)


def compact(p, geo: Geometry):
    """Compacted rows comp[Hidx, Rg, W] (uint16) and counts ncomp[Hidx, Rg]."""
    raw = p.index.view(torch.int16).numpy().view(np.uint16).astype(np.int64)
    Hidx, W = p.Hidx, raw.shape[-1]
    if p.layout_q == "BNSD":
        rows = raw.transpose(1, 0, 2, 3).reshape(Hidx, -1, W)      # [hi][b*R + i][w]
    else:
        rows = raw
    Rg = geo.Rg
    nk_row = np.full(Rg, -1, np.int64)       # -1: row belongs to no batch
    for b in range(p.B):
        lo, hi_ = geo.qoff[b], min(geo.qoff[b] + geo.nq[b], Rg)
        nk_row[lo:hi_] = geo.nk[b]
    live = nk_row >= 0
    comp = np.full((Hidx, Rg, W), NO_BLOCK, np.int64)
    ncomp = np.zeros((Hidx, Rg), np.int64)
    last = np.full((Hidx, Rg), -1, np.int64)
    bad = np.zeros((Hidx, Rg), bool)
    for w in range(W):                        # slots left to right, every row at once
        e = rows[:, :, w]
        present = e != NO_BLOCK
        ok = present & (e < nk_row[None, :]) & (e > last)
        bad |= present & ~ok
        r_h, r_g = np.nonzero(ok & live[None, :])
        comp[r_h, r_g, ncomp[r_h, r_g]] = e[r_h, r_g]
        ncomp[r_h, r_g] += 1
        last = np.where(ok, e, last)
    fl = BAD_INDEX if bool((bad & live[None, :]).any()) else 0
    return comp.astype(np.uint16), ncomp.astype(np.int32), fl


def inverted(p, geo: Geometry, comp, ncomp):
    """CSR (off[Hidx*TK+1], lst[nnz]) of the batch-local q blocks choosing each kv block."""
    Hidx, TK = p.Hidx, geo.TK
    lists = [[[] for _ in range(TK)] for _ in range(Hidx)]
    for b in range(p.B):
        for i in range(geo.nq[b]):
            gq = geo.qoff[b] + i
            if gq >= geo.Rg:
                continue
            for hi in range(Hidx):
                for x in range(int(ncomp[hi, gq])):
                    lists[hi][geo.koff[b] + int(comp[hi, gq, x])].append(i)
    off = [0]
    lst = []
    for hi in range(Hidx):
        for gk in range(TK):
            lst.extend(sorted(lists[hi][gk]))
            off.append(len(lst))
    return np.array(off, np.int32), np.array(lst, np.int32)


def packed_heads(p) -> int:
    """Query heads per forward item: g when the group shares its index row
    and g is 2, 4, 8 or 16, else 1."""
    g = p.N1 // p.N2
    return g if (p.Hidx == p.N2 and g in (2, 4, 8, 16)) else 1


def fwd_worklist(p, geo: Geometry, comp, ncomp, packed=True):
    """Item ids in execution order, and the cost of each slot id (-1: no item).
    packed=False gives the one-head-per-item list (the deterministic
    backward's q-major pass)."""
    ksl = p.BKV // 128
    g = p.N1 // p.N2
    pg = packed_heads(p) if packed else 1
    R = 128 // pg                      # query rows of one head per item
    fsub = p.BQ // R                   # items per (head or group, q block)
    nheads = p.N2 if pg > 1 else p.N1  # item heads: kv heads when packed
    Rg = geo.Rg
    cost = np.full(nheads * Rg * fsub, -1, np.int64)
    for b in range(p.B):
        for i in range(geo.nq[b]):
            gq = geo.qoff[b] + i
            if gq >= Rg:
                continue
            for hh in range(nheads):
                if pg > 1:
                    hi = hh
                else:
                    hi = hh if p.Hidx == p.N1 else hh // g
                c = 0
                for x in range(int(ncomp[hi, gq])):
                    j = int(comp[hi, gq, x])
                    c += sum(1 for s in range(ksl) if j * p.BKV + s * 128 < geo.kvlen[b])
                for qs in range(fsub):
                    if i * p.BQ + qs * R < geo.qlen[b]:
                        cost[(hh * Rg + gq) * fsub + qs] = c
    ids = np.nonzero(cost >= 0)[0]
    order = np.lexsort((ids, -cost[ids]))
    return ids[order].astype(np.int32), cost


def bwd_worklist(p, geo: Geometry, off, lst):
    nsub, ksl = p.BQ // 128, p.BKV // 128
    g = p.N1 // p.N2
    TK = geo.TK
    cost = np.full(p.N2 * TK * ksl, -1, np.int64)
    for b in range(p.B):
        for j in range(geo.nk[b]):
            gk = geo.koff[b] + j
            for h2 in range(p.N2):
                c = 0
                for h1 in range(h2 * g, (h2 + 1) * g):
                    hi = h1 if p.Hidx == p.N1 else h2
                    li = hi * TK + gk
                    for i in lst[off[li]:off[li + 1]]:
                        c += sum(1 for qs in range(nsub) if int(i) * p.BQ + qs * 128 < geo.qlen[b])
                for ks in range(ksl):
                    if j * p.BKV + ks * 128 < geo.kvlen[b]:
                        cost[(h2 * TK + gk) * ksl + ks] = c
    ids = np.nonzero(cost >= 0)[0]
    # Order (the pages' metadata step balances the load but does not say
    # how): the items above 1/512 of the list's total cost first, longest
    # first; then the rest kv head by kv head, longest first within a head
    # (costs clamped at 2^21 - 1), ties by id.  The total counts every kv
    # block at full length: the query slices of all inverse lists, times g
    # when the group shares its lists, times the kv slices per block.
    # (More than 1024 kv heads: longest first throughout.)
    sub = 0
    for hi in range(p.Hidx):
        for b in range(p.B):
            for j in range(geo.nk[b]):
                li = hi * TK + geo.koff[b] + j
                for i in lst[off[li]:off[li + 1]]:
                    sub += sum(1 for qs in range(nsub) if int(i) * p.BQ + qs * 128 < geo.qlen[b])
    total = sub * (1 if p.Hidx == p.N1 else g) * ksl
    big = total >> 9 if p.N2 <= 1024 else -1

    def key(i):
        c = int(cost[i])
        h2 = int(i) // (TK * ksl)
        if c > big:
            return (0, 0, -c, int(i))
        return (1, h2, -min(c, (1 << 21) - 1), int(i))
    order = sorted(ids.tolist(), key=key)
    return np.asarray(order, dtype=np.int32), cost


def page_flags(p, geo: Geometry) -> int:
    if p.layout_kv != "PA_BBND":
        return 0
    P = int(p.k.shape[0])
    for b in range(p.B):
        for x in range(_cdiv(geo.kvlen[b], int(p.k.shape[1]))):
            pg = int(p.block_table[b, x])
            if pg < 0 or pg >= P:
                return BAD_PAGE
    return 0


def build_all(p):
    """Every builder output, as one dict of numpy arrays."""
    geo = geometry(p)
    comp, ncomp, f1 = compact(p, geo)
    off, lst = inverted(p, geo, comp, ncomp)
    fitems, fcost = fwd_worklist(p, geo, comp, ncomp)
    fitems_1, _ = fwd_worklist(p, geo, comp, ncomp, packed=False)
    bitems, bcost = bwd_worklist(p, geo, off, lst)
    return {"geo": geo, "comp": comp, "ncomp": ncomp, "inv_off": off, "inv_list": lst,
            "fwd_items": fitems, "fwd_cost": fcost, "fwd_items_per_head": fitems_1,
            "bwd_items": bitems, "bwd_cost": bcost,
            "flags": geo.flags | f1 | page_flags(p, geo)}


def pairs(p, geo: Geometry, comp, ncomp) -> int:
    """Kept (q head, valid q token, valid kv token of a selected block) pairs."""
    g = p.N1 // p.N2
    total = 0
    for b in range(p.B):
        for i in range(geo.nq[b]):
            gq = geo.qoff[b] + i
            if gq >= geo.Rg:
                continue
            rows_i = min(p.BQ, geo.qlen[b] - i * p.BQ)
            for h1 in range(p.N1):
                hi = h1 if p.Hidx == p.N1 else h1 // g
                cols = sum(min(p.BKV, geo.kvlen[b] - int(j) * p.BKV)
                           for j in comp[hi, gq, :ncomp[hi, gq]])
                total += rows_i * cols
    return int(total)
