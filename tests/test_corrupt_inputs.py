"""Pins for the oracle's reading of data values that contradict the tensors
they describe: cu_seqlens that decrease or run past the end, seqused_kv
above the stored length or negative, block-table entries outside the page
range, and a TND index with fewer rows than the lengths need
(GenericBlockSparseAttention article: values are not checked at tiling;
the dual-length rule for seqused_kv; paged addressing).

The expected outputs are hand-derived in tests/golden/corrupt_lengths_pages.json:
with q = 0 every score is 0, so a row's softmax is uniform over the tokens
it keeps, and with v[r] = [r + 1, -2 (r + 1)] the output names the mean of
the kept kv storage rows.  A plausible slip -- clamping seqused_kv to the
storage instead of zeroing it, dropping a whole block instead of the tokens
of its bad page, flagging only selected pages, trusting an index row that
does not exist -- changes a mean, an lse or the flag word of some case.
The backward of the same inputs is pinned by central differences of the
oracle's own forward."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import builders
from workloads.gen import Problem

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "corrupt_lengths_pages.json")
CASES = json.load(open(GOLDEN))["cases"]


def _problem(name, seed=0, zero_q=True) -> Problem:
    c = CASES[name]
    lq, lkv = c["layout_q"], c["layout_kv"]
    D, dt = 2, torch.float64
    g = torch.Generator().manual_seed(seed)
    index = torch.tensor(c["index"], dtype=torch.int64).to(torch.int32).to(torch.uint16)
    cu_q = cu_kv = seq = bt = None
    if lq == "BNSD":
        B, Sq, Skv = c["B"], c["Sq"], c["Skv"]
        qshape, kshape = (B, 1, Sq, D), (B, 1, Skv, D)
        kv_rows = B * Skv
    else:
        cu_q = torch.tensor(c["cu_q"], dtype=torch.int64)
        B = cu_q.numel() - 1
        qshape = (c["Tq"], 1, D)
        if lkv == "TND":
            cu_kv = torch.tensor(c["cu_kv"], dtype=torch.int64)
            kshape = (c["Tkv"], 1, D)
            kv_rows = c["Tkv"]
        else:
            bt = torch.tensor(c["block_table"], dtype=torch.int32)
            kshape = (c["num_pages"], c["page_size"], 1, D)
            kv_rows = c["num_pages"] * c["page_size"]
    if c["seqused_kv"] is not None:
        seq = torch.tensor(c["seqused_kv"], dtype=torch.int32)
    r = torch.arange(kv_rows, dtype=dt) + 1.0
    v = torch.stack([r, -2.0 * r], 1).reshape(kshape)   # storage order == row order
    q = torch.zeros(qshape, dtype=dt) if zero_q else torch.randn(qshape, generator=g, dtype=dt)
    k = torch.randn(kshape, generator=g, dtype=dt)
    dout = torch.randn(qshape, generator=g, dtype=dt)
    return Problem(name=name, layout_q=lq, layout_kv=lkv, B=B, N1=1, N2=1, D=D, dtype=dt,
                   BQ=c["BQ"], BKV=c["BKV"], Hidx=1, scale=1.0 / math.sqrt(D), q=q, k=k, v=v,
                   dout=dout, index=index, cu_q=cu_q, cu_kv=cu_kv, seqused_kv=seq,
                   block_table=bt, page_size=c.get("page_size", 0))


def _flat_q(p, t):
    """q-layout tensor -> [q storage rows, ...] (BNSD b*Sq + t; TND token row)."""
    return t.reshape(-1, *t.shape[p.q.dim() - 1:]) if p.layout_q == "BNSD" else t[:, 0]


def _flat_kv(p, t):
    return t.reshape(-1, p.D)


@pytest.mark.parametrize("name", sorted(CASES))
def test_forward_matches_hand_derivation(name):
    c = CASES[name]
    p = _problem(name)
    o = oracle.Oracle(p)
    out, lse, fl = o.fwd()
    out_r = _flat_q(p, out)
    lse_r = lse.reshape(-1) if p.layout_q == "BNSD" else lse[:, 0]
    for row in c["rows"]:
        n = len(row["kv_rows"])
        m = float(row["mean"])
        if n:   # the fixture's mean is that of (r + 1) over its rows
            assert m == pytest.approx(sum(x + 1 for x in row["kv_rows"]) / n, abs=0)
        got = out_r[row["q_row"]]
        assert torch.allclose(got, torch.tensor([m, -2.0 * m], dtype=torch.float64),
                              atol=1e-12, rtol=0), (row, got)
        got_lse = float(lse_r[row["q_row"]])
        if n:
            assert abs(got_lse - math.log(n)) <= 1e-12, (row, got_lse)
        else:
            assert got_lse == float("-inf"), (row, got_lse)
    assert (fl | o.scan_flags()) == c["flags"]
    assert o.scan_flags() == c["flags"]


@pytest.mark.parametrize("name", sorted(CASES))
def test_builders_agree_on_flags_and_rows(name):
    """The builder oracle raises the same flag word, and its rows reach only
    the query blocks that have an index row."""
    c = CASES[name]
    B = builders.build_all(_problem(name))
    assert B["flags"] == c["flags"]


@pytest.mark.parametrize("name", sorted(CASES))
def test_undefined_rows_are_not_enumerated(name):
    """Query rows of no valid batch are not rows of the problem, and kv rows of
    no valid batch or bad page are not rows the backward owns."""
    c = CASES[name]
    p = _problem(name)
    o = oracle.Oracle(p)
    rows = o.q_rows_all()
    if p.layout_q == "TND":
        cu = p.cu_q.tolist()
        stored = {cu[b] + t for b, _, t in rows.tolist()}
    else:
        stored = {b * p.q.shape[2] + t for b, _, t in rows.tolist()}
    assert stored.isdisjoint(c["undefined_q_rows"])
    assert stored == {r["q_row"] for r in c["rows"]}


@pytest.mark.parametrize("name", sorted(CASES))
def test_backward_zero_rows_and_finite_differences(name):
    """dK/dV of kv rows nobody keeps are exactly 0, dQ of rows that keep
    nothing is exactly 0, and the gradients equal central differences of
    L = sum(dOut * out) through the oracle's forward (random q, so the
    scores are no longer all equal)."""
    c = CASES[name]
    p = _problem(name, seed=7, zero_q=False)
    o = oracle.Oracle(p)
    out, lse, _ = o.fwd()
    dq, dk, dv, _ = o.bwd(out, p.dout, lse)
    for r in c["zero_grad_kv_rows"]:
        assert torch.all(_flat_kv(p, dk)[r] == 0) and torch.all(_flat_kv(p, dv)[r] == 0)
    for row in c["rows"]:
        if not row["kv_rows"]:
            assert torch.all(_flat_q(p, dq)[row["q_row"]] == 0)

    def loss(**kw):
        o2, _, _ = oracle.Oracle(p, **kw).fwd()
        return float((o2 * p.dout).sum())

    eps = 1e-6
    for tname, grad in (("q", dq), ("k", dk), ("v", dv)):
        base = getattr(p, tname)
        for pos in np.ndindex(*base.shape):
            args = {"q": p.q, "k": p.k, "v": p.v}
            plus, minus = base.clone(), base.clone()
            plus[pos] += eps
            minus[pos] -= eps
            args[tname] = plus
            lp = loss(**args)
            args[tname] = minus
            lm = loss(**args)
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - float(grad[pos])) <= 1e-6 * max(1.0, abs(fd)), (tname, pos, fd,
                                                                           float(grad[pos]))
