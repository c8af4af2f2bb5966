"""Seeded problem generator.

Every random draw is seeded with ``1000 * config + k`` where k names the
stream: 1 q, 2 k, 3 v, 4 dout, 5 index, 6 lengths, 7 block table.  Float
tensors are N(0, 1) in fp32 rounded to the compute dtype; integer structure
(lengths, index rows, page permutation) comes from numpy's PCG64.

Index format (BlitzSparseAttention, "sabi" section): uint16 rows of
batch-local KV block ids, ascending, right-padded with 0xFFFF.  BNSD uses
``[B, Hidx, ceil(Sq/BQ), W]``; TND uses the GenericBlockSparseAttention
packed-row form ``[Hidx, totalQBlocks, W]`` with the rows of batch b
starting after the ``ceil(qlen/BQ)`` rows of every earlier batch.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Callable, List, Optional

import numpy as np
import torch

NO_BLOCK = 0xFFFF


@dataclass
class Problem:
    name: str
    layout_q: str            # 'BNSD' | 'TND'
    layout_kv: str           # 'BNSD' | 'TND' | 'PA_BBND'
    B: int
    N1: int
    N2: int
    D: int
    dtype: torch.dtype
    BQ: int
    BKV: int
    Hidx: int
    scale: float
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    dout: torch.Tensor
    index: torch.Tensor      # uint16
    cu_q: Optional[torch.Tensor] = None        # int64 [B+1]
    cu_kv: Optional[torch.Tensor] = None       # int64 [B+1]
    seqused_kv: Optional[torch.Tensor] = None  # int32 [B]
    block_table: Optional[torch.Tensor] = None  # int32 [B, max_pages]
    page_size: int = 0
    lens_q: List[int] = field(default_factory=list)
    lens_kv: List[int] = field(default_factory=list)
    causal: bool = False     # kv token u visible to query row t iff u <= t + kvlen - qlen
    out_dtype: Optional[torch.dtype] = None  # out / dout dtype when q, k, v are 8-bit

    @property
    def odtype(self) -> torch.dtype:
        """dtype of out (and dout): the input dtype, or out_dtype for FP8 inputs."""
        return self.out_dtype if self.out_dtype is not None else self.dtype

    @property
    def W(self) -> int:
        return int(self.index.shape[-1])

    def describe(self) -> dict:
        return {"name": self.name, "layout_q": self.layout_q, "layout_kv": self.layout_kv,
                "B": self.B, "N1": self.N1, "N2": self.N2, "D": self.D,
                "dtype": str(self.dtype).replace("torch.", ""),
                "block_shape": [self.BQ, self.BKV], "Hidx": self.Hidx, "W": self.W,
                "lens_q": self.lens_q, "lens_kv": self.lens_kv, "page_size": self.page_size,
                "causal": self.causal}


# ----------------------------------------------------------------------------
# row patterns: (rng, i, nq_b, nk_b) -> list of kv block ids (any order)
# ----------------------------------------------------------------------------
def pat_random_k(rng, i, nq, nk):
    """k ~ U{1..nk}, a uniform k-subset."""
    if nk == 0:
        return []
    k = int(rng.integers(1, nk + 1))
    return list(rng.choice(nk, size=k, replace=False))


def pat_fraction_diag(frac):
    """ceil(frac*nk) blocks (>= 1), always the diagonal block i, rest uniform."""
    def f(rng, i, nq, nk):
        if nk == 0:
            return []
        k = max(1, math.ceil(frac * nk))
        sel = {i} if i < nk else set()
        others = [j for j in range(nk) if j not in sel]
        need = max(0, k - len(sel))
        if need and others:
            sel |= set(int(x) for x in rng.choice(others, size=min(need, len(others)), replace=False))
        return list(sel)
    return f


def pat_dense(rng, i, nq, nk):
    return list(range(nk))


def pat_causal(rng, i, nq, nk):
    """Every block a causal row can reach (query and kv blocks of equal size,
    the kv sequence ending where the query sequence ends)."""
    return list(range(min(nk, i + 1 + max(0, nk - nq))))


def pat_causal_blocks(BQ, BKV):
    """Every kv block of BKV tokens that a causal row of query block i (BQ
    rows) can reach, with query and kv sequences of one length."""
    def f(rng, i, nq, nk):
        return list(range(min(nk, (i * BQ + BQ - 1) // BKV + 1)))
    return f


def pat_sink_diag_random(extra):
    """block 0, the diagonal block i and `extra` distinct random blocks from [1, i-1]."""
    def f(rng, i, nq, nk):
        top = min(i, nk - 1)
        if top < 0:
            return []
        cand = list(range(1, top))
        if len(cand) <= extra:
            return list(range(0, top + 1))
        pick = rng.choice(len(cand), size=extra, replace=False)
        return [0, top] + [cand[int(p)] for p in pick]
    return f


def pat_topk(k):
    """min(k, nk) blocks chosen uniformly (the top-k of i.i.d. random scores)."""
    def f(rng, i, nq, nk):
        if nk == 0:
            return []
        return list(rng.choice(nk, size=min(k, nk), replace=False))
    return f


def pat_density(density, min_keep=0):
    """each block kept independently with probability `density`."""
    def f(rng, i, nq, nk):
        keep = [j for j in range(nk) if rng.random() < density]
        if len(keep) < min_keep and nk:
            keep = list(rng.choice(nk, size=min(min_keep, nk), replace=False))
        return keep
    return f


# ----------------------------------------------------------------------------
def _randn(shape, seed, dtype):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(dtype)


def make_problem(*, name="custom", layout_q="BNSD", layout_kv="BNSD", B=1, N1=2, N2=2, D=64,
                 dtype=torch.bfloat16, BQ=128, BKV=128, lens_q=None, lens_kv=None,
                 Sq=None, Skv=None, kv_storage=None, Hidx=None, W=None,
                 pattern: Callable = pat_random_k, page_size=128, extra_pages=0,
                 use_seqused_kv=None, seed_base=0, scale=None, max_pages=None,
                 row_hook: Optional[Callable] = None, causal: bool = False,
                 out_dtype: Optional[torch.dtype] = None) -> Problem:
    """Build one seeded problem.

    lens_q / lens_kv: per-batch valid lengths (TND q: the stored lengths).
    Sq / Skv: BNSD storage lengths (default: max length).
    kv_storage: TND kv stored lengths (default lens_kv; >= lens_kv, then
    seqused_kv carries the used lengths).
    row_hook(rng, b, hi, i, row_list) -> list[int]: lets a test write raw
    slot values (0xFFFF in mid-row, out-of-range or repeated ids).
    dtype torch.float8_e4m3fn: q, k, v are N(0,1) rounded to e4m3 (the
    GenericBlockSparseAttention FP8 inputs); out_dtype (default bf16) is the
    dtype of out and dout.
    """
    if dtype == torch.float8_e4m3fn and out_dtype is None:
        out_dtype = torch.bfloat16
    odt = out_dtype if out_dtype is not None else dtype
    s = seed_base
    lens_q = list(lens_q) if lens_q is not None else [Sq] * B
    lens_kv = list(lens_kv) if lens_kv is not None else list(lens_q)
    assert len(lens_q) == B and len(lens_kv) == B
    Hidx = N1 if Hidx is None else Hidx
    scale = (1.0 / math.sqrt(D)) if scale is None else scale

    cu_q = cu_kv = seqused = block_table = None
    if layout_q == "BNSD":
        Sq = Sq if Sq is not None else max(lens_q)
        assert all(l == Sq for l in lens_q), "BNSD query rows are all valid"
        q = _randn((B, N1, Sq, D), s + 1, dtype)
        dout = _randn((B, N1, Sq, D), s + 4, odt)
    else:
        Tq = sum(lens_q)
        cu_q = torch.tensor([0] + list(np.cumsum(lens_q)), dtype=torch.int64)
        q = _randn((Tq, N1, D), s + 1, dtype)
        dout = _randn((Tq, N1, D), s + 4, odt)

    if layout_kv == "BNSD":
        Skv = Skv if Skv is not None else max(lens_kv)
        k = _randn((B, N2, Skv, D), s + 2, dtype)
        v = _randn((B, N2, Skv, D), s + 3, dtype)
        if use_seqused_kv or (use_seqused_kv is None and any(l != Skv for l in lens_kv)):
            seqused = torch.tensor(lens_kv, dtype=torch.int32)
    elif layout_kv == "TND":
        kv_storage = list(kv_storage) if kv_storage is not None else list(lens_kv)
        cu_kv = torch.tensor([0] + list(np.cumsum(kv_storage)), dtype=torch.int64)
        Tkv = int(cu_kv[-1])
        k = _randn((Tkv, N2, D), s + 2, dtype)
        v = _randn((Tkv, N2, D), s + 3, dtype)
        if use_seqused_kv or (use_seqused_kv is None and kv_storage != lens_kv):
            seqused = torch.tensor(lens_kv, dtype=torch.int32)
    else:  # PA_BBND
        pages_b = [math.ceil(l / page_size) for l in lens_kv]
        P = sum(pages_b) + extra_pages
        max_pages = max_pages if max_pages is not None else max(1, max(pages_b))
        rng_bt = np.random.default_rng(s + 7)
        perm = rng_bt.permutation(P)
        bt = np.zeros((B, max_pages), dtype=np.int32)
        o = 0
        for b in range(B):
            bt[b, :pages_b[b]] = perm[o:o + pages_b[b]]
            o += pages_b[b]
        block_table = torch.from_numpy(bt)
        k = _randn((P, page_size, N2, D), s + 2, dtype)
        v = _randn((P, page_size, N2, D), s + 3, dtype)
        seqused = torch.tensor(lens_kv, dtype=torch.int32)

    # ---- the block index ----
    rng = np.random.default_rng(s + 5)
    nq = [math.ceil(l / BQ) for l in lens_q]
    nk = [math.ceil(l / BKV) for l in lens_kv]
    rows = []   # (b, hi, i, list)
    for b in range(B):
        for hi in range(Hidx):
            for i in range(nq[b]):
                sel = sorted(set(int(x) for x in pattern(rng, i, nq[b], nk[b])))
                if row_hook is not None:
                    sel = row_hook(rng, b, hi, i, sel)
                rows.append((b, hi, i, sel))
    if W is None:
        W = max([len(r[3]) for r in rows] + [1])
    if layout_q == "BNSD":
        idx = np.full((B, Hidx, math.ceil(Sq / BQ), W), NO_BLOCK, dtype=np.uint16)
        for b, hi, i, sel in rows:
            idx[b, hi, i, :len(sel)] = sel[:W]
    else:
        off = [0] + list(np.cumsum(nq))
        idx = np.full((Hidx, int(off[-1]), W), NO_BLOCK, dtype=np.uint16)
        for b, hi, i, sel in rows:
            idx[hi, off[b] + i, :len(sel)] = sel[:W]
    index = torch.from_numpy(idx.view(np.int16).copy()).view(torch.uint16)

    return Problem(name=name, layout_q=layout_q, layout_kv=layout_kv, B=B, N1=N1, N2=N2, D=D,
                   dtype=dtype, BQ=BQ, BKV=BKV, Hidx=Hidx, scale=scale, q=q, k=k, v=v,
                   dout=dout, index=index, cu_q=cu_q, cu_kv=cu_kv, seqused_kv=seqused,
                   block_table=block_table, page_size=(page_size if layout_kv == "PA_BBND" else 0),
                   lens_q=lens_q, lens_kv=lens_kv, causal=causal, out_dtype=out_dtype)


# ----------------------------------------------------------------------------
# the five workloads
# ----------------------------------------------------------------------------
def _lens(seed, B, lo, hi):
    rng = np.random.default_rng(seed)
    return [int(x) for x in rng.integers(lo, hi + 1, size=B)]


def make_config(c: int, batch: int | None = None, causal: bool = False, fp8: bool = False,
                shared_rows: bool = False, per_head_rows: bool = False,
                heads: int | None = None) -> Problem:
    """C1..C5: the five workload shapes (see the module docstring for seeds).

    `batch` and `heads` (N1 = N2) override the batch and head count of the
    BNSD shapes C3 and C4 (smaller cases of the same kernels for profiler
    captures).  `causal` turns C3 into its
    causal variant: the causal mask with the lower-triangular block index;
    `fp8` gives C3 e4m3 q, k, v (bf16 out), the same N(0,1) draws rounded to
    e4m3.  `shared_rows` (C2, C5) draws one index row per GQA group instead
    of one per query head (Hidx = N2, the GenericBlockSparseAttention
    isPackedGQA pattern); `per_head_rows` then copies each group's row to
    every query head of the group (Hidx = N1: the same selection, stated per
    head)."""
    if (shared_rows or per_head_rows) and c not in (2, 5):
        raise ValueError("the shared-row variants are defined for C2 and C5")
    if per_head_rows and not shared_rows:
        raise ValueError("per_head_rows copies the rows of the shared-row variant")
    if shared_rows:
        q = make_config_shared(c)
        if per_head_rows:
            g = q.N1 // q.N2
            q.index = q.index.view(torch.int16).repeat_interleave(g, dim=0).view(torch.uint16)
            q.Hidx = q.N1
            q.name += "-per-head-rows"
        return q
    if fp8 and c != 3:
        raise ValueError("the FP8 variant is defined for C3 only")
    if (batch is not None or heads is not None) and c not in (3, 4):
        raise ValueError("batch / head overrides apply to C3 and C4 only")
    if causal and c != 3:
        raise ValueError("the causal variant is defined for C3 only")
    s = 1000 * c
    if c == 1:
        return make_problem(name="C1", layout_q="BNSD", layout_kv="BNSD", B=1, N1=2, N2=2, D=64,
                            Sq=512, BQ=128, BKV=128, W=4, pattern=pat_random_k, seed_base=s)
    if c == 2:
        lens = _lens(s + 6, 4, 256, 3072)
        return make_problem(name="C2", layout_q="TND", layout_kv="TND", B=4, N1=16, N2=4, D=128,
                            lens_q=lens, lens_kv=lens, BQ=128, BKV=128,
                            pattern=pat_fraction_diag(0.25), W=max(math.ceil(l / 128) for l in lens),
                            seed_base=s)
    if c == 3:
        return make_problem(name="C3-causal" if causal else "C3", layout_q="BNSD", layout_kv="BNSD",
                            B=batch or 2, N1=heads or 32, N2=heads or 32, D=128, Sq=8192, BQ=128,
                            BKV=512, W=16,
                            pattern=pat_causal_blocks(128, 512) if causal else pat_dense,
                            seed_base=s, causal=causal,
                            dtype=torch.float8_e4m3fn if fp8 else torch.bfloat16)
    if c == 4:
        return make_problem(name="C4", layout_q="BNSD", layout_kv="BNSD", B=batch or 1, N1=heads or 24,
                            N2=heads or 24, D=128,
                            Sq=32768, BQ=128, BKV=128, W=256, pattern=pat_sink_diag_random(14),
                            seed_base=s)
    if c == 5:
        lens = _lens(s + 6, 8, 512, 4096)
        return make_problem(name="C5", layout_q="TND", layout_kv="PA_BBND", B=8, N1=32, N2=8, D=128,
                            dtype=torch.float16, lens_q=lens, lens_kv=lens, BQ=128, BKV=128,
                            page_size=128, max_pages=32, W=8, pattern=pat_topk(8), seed_base=s)
    raise ValueError(f"unknown config C{c}")


def make_config_shared(c: int) -> Problem:
    """C2 / C5 with one index row per kv-head group (Hidx = N2), same seeds."""
    s = 1000 * c
    if c == 2:
        lens = _lens(s + 6, 4, 256, 3072)
        return make_problem(name="C2-shared-rows", layout_q="TND", layout_kv="TND", B=4, N1=16, N2=4,
                            Hidx=4, D=128, lens_q=lens, lens_kv=lens, BQ=128, BKV=128,
                            pattern=pat_fraction_diag(0.25), W=max(math.ceil(l / 128) for l in lens),
                            seed_base=s)
    if c == 5:
        lens = _lens(s + 6, 8, 512, 4096)
        return make_problem(name="C5-shared-rows", layout_q="TND", layout_kv="PA_BBND", B=8, N1=32,
                            N2=8, Hidx=8, D=128, dtype=torch.float16, lens_q=lens, lens_kv=lens,
                            BQ=128, BKV=128, page_size=128, max_pages=32, W=8, pattern=pat_topk(8),
                            seed_base=s)
    raise ValueError(f"no shared-row variant of C{c}")


CONFIGS = {f"C{c}": c for c in range(1, 6)}
