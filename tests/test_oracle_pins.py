"""Pins for the CPU oracle: each check ties the oracle to something other than
itself -- the worked example printed on the BlitzSparseAttention page, closed
forms, torch library routines on the equivalent dense masked problem,
finite differences, and invariances the definition implies."""
import math
import os
import zlib

import numpy as np
import pytest
import torch

import oracle
import workloads
from workloads.gen import (make_problem, pat_causal, pat_dense, pat_density, pat_fraction_diag,
                           pat_random_k, pat_topk)
from tests import torch_reference as tr

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    vals = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()
            vals[k] = v
    return vals


# ---------------------------------------------------------------- worked example
def test_all_ones_worked_example():
    """BlitzSparseAttention page, call example: all-ones fp16 [1,8,512,128],
    dense sabi [1,8,4,4] -> out == 1 (0x3C00) and lse == ln(512) + sqrt(128)."""
    g = _golden("all_ones_bnsd.txt")
    B, N, S, D = (int(g[k]) for k in ("B", "N", "S", "D"))
    p = make_problem(B=B, N1=N, N2=N, D=D, Sq=S, dtype=torch.float16, BQ=int(g["block_q"]),
                     BKV=int(g["block_kv"]), pattern=pat_dense, W=S // int(g["block_kv"]))
    p.q.fill_(1.0); p.k.fill_(1.0); p.v.fill_(1.0)
    rows = np.array([[0, h, t] for h in (0, N - 1) for t in (0, 1, 255, S - 1)], np.int64)
    out, lse, fl = oracle.Oracle(p).fwd_rows(rows)
    closed = math.log(int(g["expected_lse_closed_form_S"])) + math.sqrt(int(g["expected_lse_closed_form_D"]))
    assert fl == 0
    assert np.allclose(out, 1.0, atol=1e-13, rtol=0)
    assert np.allclose(lse, closed, atol=1e-12, rtol=0)
    assert abs(lse[0] - float(g["expected_lse_quoted"])) < 1e-4
    # the page's device value is within fp16-era accumulation error of it
    assert abs(lse[0] - float(g["device_lse_printed"])) < 2e-3
    assert np.float16(out[0, 0]).view(np.uint16) == int(g["device_out0_printed_fp16_bits"], 16)


@pytest.mark.parametrize("S,D", [(128, 64), (384, 128), (1000, 64)])
def test_all_ones_closed_form_any_size(S, D):
    """Uniform scores: lse = ln(#selected tokens) + D*scale, out = v."""
    p = make_problem(B=1, N1=1, N2=1, D=D, Sq=S, BQ=128, BKV=128, pattern=pat_dense)
    p.q.fill_(1.0); p.k.fill_(1.0)
    p.v.copy_(torch.arange(D, dtype=torch.float32).to(p.v.dtype).expand_as(p.v))
    rows = np.array([[0, 0, t] for t in (0, S // 2, S - 1)], np.int64)
    out, lse, _ = oracle.Oracle(p).fwd_rows(rows)
    assert np.allclose(lse, math.log(S) + D * p.scale, atol=1e-12)
    assert np.allclose(out, np.arange(D)[None, :], atol=1e-12)


# ------------------------------------------------------ library: dense / masked
def _compare_fwd(p, atol=1e-11):
    o = oracle.Oracle(p)
    out, lse, fl = o.fwd()
    ref = tr.attention(p)
    rout, rlse = tr.to_q_layout(p, ref, 0), tr.to_q_layout(p, ref, 1)
    assert fl == 0
    assert torch.allclose(out, rout, atol=atol, rtol=0)
    fin = torch.isfinite(rlse)
    assert torch.equal(fin, torch.isfinite(lse))
    assert torch.allclose(lse[fin], rlse[fin], atol=atol, rtol=0)
    assert torch.all(lse[~fin] == float("-inf"))
    return out, lse


def test_dense_index_is_softmax_attention():
    """Fully dense index == torch scaled_dot_product_attention (fp64)."""
    p = make_problem(B=2, N1=3, N2=3, D=64, Sq=256, BQ=128, BKV=128, pattern=pat_dense, seed_base=11)
    out, lse = oracle.Oracle(p).fwd()[:2]
    q, k, v = p.q.double(), p.k.double(), p.v.double()
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=p.scale)
    assert torch.allclose(out, ref, atol=1e-12, rtol=0)
    rl = torch.logsumexp(p.scale * q @ k.transpose(-1, -2), -1)
    assert torch.allclose(lse, rl, atol=1e-12, rtol=0)


CASES = {
    "bnsd_random": dict(layout_q="BNSD", layout_kv="BNSD", B=2, N1=2, N2=2, D=64, Sq=384,
                        pattern=pat_random_k),
    "bnsd_ragged_kv": dict(layout_q="BNSD", layout_kv="BNSD", B=2, N1=2, N2=1, D=64, Sq=300,
                           lens_kv=[300, 170], Skv=300, pattern=pat_density(0.5, 1)),
    "bnsd_blocks": dict(layout_q="BNSD", layout_kv="BNSD", B=1, N1=2, N2=2, D=32, Sq=640,
                        BQ=256, BKV=128, pattern=pat_density(0.4, 1)),
    "tnd_gqa": dict(layout_q="TND", layout_kv="TND", B=3, N1=4, N2=2, D=64,
                    lens_q=[130, 300, 77], lens_kv=[200, 129, 256], pattern=pat_fraction_diag(0.5)),
    "tnd_shared_rows": dict(layout_q="TND", layout_kv="TND", B=2, N1=4, N2=2, Hidx=2, D=64,
                            lens_q=[256, 140], lens_kv=[256, 140], pattern=pat_random_k),
    "tnd_seqused": dict(layout_q="TND", layout_kv="TND", B=2, N1=2, N2=2, D=64,
                        lens_q=[200, 90], lens_kv=[150, 60], kv_storage=[260, 100],
                        pattern=pat_random_k),
    "paged": dict(layout_q="TND", layout_kv="PA_BBND", B=3, N1=4, N2=2, D=64,
                  lens_q=[300, 129, 64], lens_kv=[300, 129, 64], page_size=128, extra_pages=2,
                  pattern=pat_topk(2)),
    "big_blocks": dict(layout_q="TND", layout_kv="TND", B=2, N1=2, N2=2, D=64, BQ=512, BKV=256,
                       lens_q=[700, 300], lens_kv=[900, 300], pattern=pat_random_k),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_sparse_equals_masked_dense(name):
    """Block-sparse == dense attention with -inf outside the selected blocks
    (bool-mask form of the same pattern, torch matmul/softmax/logsumexp)."""
    p = make_problem(seed_base=zlib.crc32(name.encode()) % 997, **CASES[name])
    _compare_fwd(p)


def test_rows_sum_to_one_and_empty_rows():
    """Softmax rows sum to 1 (v with a constant feature); a row with no
    accepted block gives out 0 and lse -inf."""
    def hook(rng, b, hi, i, sel):
        return [] if (i == 1 and hi == 0) else sel
    p = make_problem(B=1, N1=2, N2=2, D=64, Sq=512, pattern=pat_random_k, row_hook=hook, seed_base=5)
    p.v[..., 0] = 1.0
    out, lse, fl = oracle.Oracle(p).fwd()
    assert fl == 0
    empty = torch.zeros_like(lse, dtype=torch.bool)
    empty[0, 0, 128:256] = True
    assert torch.all(lse[empty] == float("-inf"))
    assert torch.all(out[0, 0, 128:256] == 0)
    assert torch.allclose(out[..., 0][~empty], torch.ones(()).double(), atol=1e-13)


# ------------------------------------------------------------- invariances
def test_gqa_equals_repeated_mha():
    p = make_problem(layout_q="TND", layout_kv="TND", B=2, N1=4, N2=2, D=64, lens_q=[200, 140],
                     pattern=pat_random_k, seed_base=21)
    out, lse, _ = oracle.Oracle(p).fwd()
    k2 = p.k.repeat_interleave(2, 1)
    v2 = p.v.repeat_interleave(2, 1)
    p2 = make_problem(layout_q="TND", layout_kv="TND", B=2, N1=4, N2=4, D=64, lens_q=[200, 140],
                      pattern=pat_random_k, seed_base=21)
    p2.k, p2.v, p2.index = k2, v2, p.index
    out2, lse2, _ = oracle.Oracle(p2).fwd()
    assert torch.allclose(out, out2, atol=1e-14) and torch.equal(lse, lse2)


def test_tnd_equals_independent_bnsd():
    lens = [130, 256, 77]
    p = make_problem(layout_q="TND", layout_kv="TND", B=3, N1=2, N2=2, D=64, lens_q=lens,
                     pattern=pat_random_k, seed_base=31)
    out, lse, _ = oracle.Oracle(p).fwd()
    cu = p.cu_q.tolist()
    idx = p.index.view(torch.int16)
    qoff = 0
    for b, L in enumerate(lens):
        nq = -(-L // 128)
        pb = make_problem(B=1, N1=2, N2=2, D=64, Sq=L, pattern=pat_dense, seed_base=0)
        pb.q = p.q[cu[b]:cu[b + 1]].transpose(0, 1).unsqueeze(0).contiguous()
        pb.k = p.k[cu[b]:cu[b + 1]].transpose(0, 1).unsqueeze(0).contiguous()
        pb.v = p.v[cu[b]:cu[b + 1]].transpose(0, 1).unsqueeze(0).contiguous()
        pb.index = idx[:, qoff:qoff + nq].unsqueeze(0).contiguous().view(torch.uint16)
        ob, lb, _ = oracle.Oracle(pb).fwd()
        assert torch.allclose(ob[0].transpose(0, 1), out[cu[b]:cu[b + 1]], atol=1e-14)
        assert torch.equal(lb[0].transpose(0, 1), lse[cu[b]:cu[b + 1]])
        qoff += nq


def test_paged_equals_contiguous():
    lens = [300, 129, 64]
    p = make_problem(layout_q="TND", layout_kv="PA_BBND", B=3, N1=2, N2=2, D=64, lens_q=lens,
                     page_size=128, extra_pages=3, pattern=pat_random_k, seed_base=41)
    out, lse, _ = oracle.Oracle(p).fwd()
    # gather the pages into a contiguous TND kv
    ks, vs = [], []
    for b, L in enumerate(lens):
        pages = p.block_table[b, :-(-L // 128)].long()
        ks.append(p.k[pages].reshape(-1, 2, 64)[:L])
        vs.append(p.v[pages].reshape(-1, 2, 64)[:L])
    p2 = make_problem(layout_q="TND", layout_kv="TND", B=3, N1=2, N2=2, D=64, lens_q=lens,
                      pattern=pat_random_k, seed_base=41)
    p2.k, p2.v, p2.index, p2.q = torch.cat(ks), torch.cat(vs), p.index, p.q
    out2, lse2, _ = oracle.Oracle(p2).fwd()
    assert torch.allclose(out, out2, atol=1e-14) and torch.equal(lse, lse2)


def test_invalid_entries_are_ignored_and_flagged():
    """Out-of-range, repeated and descending entries and 0xFFFF mid-row:
    flagged, and the result equals the row with those slots cleared."""
    def hook(rng, b, hi, i, sel):
        if i == 0 and hi == 0:
            return [1, 0xFFFF, 1, 0, 3, 9]      # 1 ok, skip, dup, desc, 3 ok, 9 out of range
        return sel
    p = make_problem(B=1, N1=2, N2=2, D=64, Sq=512, W=6, pattern=pat_random_k, row_hook=hook, seed_base=7)
    o = oracle.Oracle(p)
    out, lse, fl = o.fwd()
    assert fl & oracle.BAD_INDEX
    assert o.scan_flags() == oracle.BAD_INDEX
    clean = p.index.view(torch.int16).clone().view(torch.uint16)
    row = np.full(6, 0xFFFF, np.uint16); row[0], row[1] = 1, 3
    clean[0, 0, 0] = torch.from_numpy(row.view(np.int16)).view(torch.uint16)
    p.index = clean
    out2, lse2, fl2 = oracle.Oracle(p).fwd()
    assert fl2 == 0
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


# ------------------------------------------------------------------ backward
BWD_CASES = ["bnsd_random", "tnd_gqa", "tnd_shared_rows", "paged", "bnsd_ragged_kv"]


@pytest.mark.parametrize("name", BWD_CASES)
def test_backward_equals_autograd(name):
    """dq/dk/dv == torch autograd of sum(dOut * out) on the dense masked problem."""
    p = make_problem(seed_base=zlib.crc32(name.encode()) % 991, **CASES[name])
    o = oracle.Oracle(p)
    out, lse, _ = o.fwd()
    dq, dk, dv, fl = o.bwd(out, p.dout, lse)
    rq, rk, rv = tr.grads(p, p.dout)
    assert fl == 0
    for a, r in ((dq, rq), (dk, rk), (dv, rv)):
        assert torch.allclose(a, r, atol=1e-10, rtol=0), (a - r).abs().max()


def test_backward_finite_differences():
    """Central differences of L = sum(dOut * out) (oracle forward only),
    4x4 blocks on a tiny sequence (the oracle accepts any block shape)."""
    p = make_problem(layout_q="TND", layout_kv="TND", B=2, N1=2, N2=1, D=8, BQ=4, BKV=4,
                     lens_q=[13, 9], lens_kv=[11, 16], pattern=pat_random_k, seed_base=3,
                     dtype=torch.float64)
    dout = p.dout.double()

    def loss(q, k, v):
        out, _, _ = oracle.Oracle(p, q=q, k=k, v=v).fwd()
        return float((out * dout).sum())

    o = oracle.Oracle(p)
    out, lse, _ = o.fwd()
    dq, dk, dv, _ = o.bwd(out, dout, lse)
    rng = np.random.default_rng(0)
    eps = 1e-6
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        base = getattr(p, name).double()
        for _ in range(6):
            pos = tuple(int(rng.integers(0, s)) for s in base.shape)
            plus, minus = base.clone(), base.clone()
            plus[pos] += eps
            minus[pos] -= eps
            args = {"q": p.q.double(), "k": p.k.double(), "v": p.v.double()}
            args[name] = plus
            lp = loss(**args)
            args[name] = minus
            lm = loss(**args)
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - float(grad[pos])) <= 1e-6 * max(1.0, abs(fd)), (name, pos, fd, float(grad[pos]))


def test_backward_invariants():
    """sum_u dK_u = 0 (rows of dS sum to 0 with the exact out) and
    sum_u dV_u = sum over non-empty rows of dOut, per (batch, kv head)."""
    p = make_problem(B=2, N1=2, N2=2, D=32, Sq=384, pattern=pat_random_k, seed_base=17)
    o = oracle.Oracle(p)
    out, lse, _ = o.fwd()
    dq, dk, dv, _ = o.bwd(out, p.dout, lse)
    assert torch.allclose(dk.sum(2), torch.zeros(()).double(), atol=1e-10)
    live = torch.isfinite(lse).unsqueeze(-1)
    assert torch.allclose(dv.sum(2), (p.dout.double() * live).sum(2), atol=1e-10)


@pytest.mark.parametrize("c", [1, 2])
def test_config_rows_match_reference(c):
    """Workload C1 in full and sampled C2 rows match the library reference."""
    p = workloads.make_config(c)
    if c == 1:
        _compare_fwd(p)
        return
    o = oracle.Oracle(p)
    rows = o.q_rows_all()[np.random.default_rng(1).choice(len(o.q_rows_all()), 64, replace=False)]
    out, lse, fl = o.fwd_rows(rows)
    ref = tr.attention(p)
    rout, rlse = tr.to_q_layout(p, ref, 0), tr.to_q_layout(p, ref, 1)
    assert fl == 0
    assert np.allclose(out, o.gather_q(rout, rows).numpy(), atol=1e-11)
    assert np.allclose(lse, o.gather_q(rlse, rows).numpy(), atol=1e-11)


# ------------------------------------------------------------ causal mask
def test_causal_dense_is_sdpa_causal():
    """Dense index + causal mask == torch scaled_dot_product_attention with
    is_causal=True (fp64), forward and, through autograd, backward."""
    p = make_problem(B=1, N1=2, N2=2, D=32, Sq=200, BQ=64, BKV=64, pattern=pat_dense, seed_base=17,
                     causal=True)
    o = oracle.Oracle(p)
    out, lse, fl = o.fwd()
    assert fl == 0
    q, k, v = (t.double().requires_grad_() for t in (p.q, p.k, p.v))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=p.scale, is_causal=True)
    assert torch.allclose(out, ref.detach(), atol=1e-12, rtol=0)
    dq, dk, dv, _ = o.bwd(out, p.dout, lse)
    ref.backward(p.dout.double())
    for a, r in ((dq, q.grad), (dk, k.grad), (dv, v.grad)):
        assert torch.allclose(a, r, atol=1e-10, rtol=0), (a - r).abs().max()


def test_causal_short_query_is_the_tail_of_a_square_problem():
    """With fewer query than kv tokens the mask is aligned to the end of the
    kv sequence: the result equals the last rows of the square causal problem
    whose last query rows are these."""
    n_kv, n_q = 150, 40
    sq = make_problem(layout_q="TND", layout_kv="TND", B=1, N1=2, N2=1, D=16, BQ=32, BKV=32,
                      lens_q=[n_kv], lens_kv=[n_kv], pattern=pat_dense, seed_base=23, causal=True,
                      dtype=torch.float64)
    short = make_problem(layout_q="TND", layout_kv="TND", B=1, N1=2, N2=1, D=16, BQ=32, BKV=32,
                         lens_q=[n_q], lens_kv=[n_kv], pattern=pat_dense, seed_base=23, causal=True,
                         dtype=torch.float64)
    short.q = sq.q[n_kv - n_q:].clone()
    short.k, short.v = sq.k, sq.v
    out_sq, lse_sq, _ = oracle.Oracle(sq).fwd()
    out_sh, lse_sh, fl = oracle.Oracle(short).fwd()
    assert fl == 0
    assert torch.allclose(out_sh, out_sq[n_kv - n_q:], atol=1e-13, rtol=0)
    assert torch.allclose(lse_sh, lse_sq[n_kv - n_q:], atol=1e-13, rtol=0)


CAUSAL_CASES = {
    "bnsd_causal_sparse": dict(layout_q="BNSD", layout_kv="BNSD", B=2, N1=2, N2=1, D=32, Sq=300,
                               pattern=pat_random_k),
    "tnd_causal_short_q": dict(layout_q="TND", layout_kv="TND", B=2, N1=2, N2=2, D=32,
                               lens_q=[70, 200], lens_kv=[260, 200], pattern=pat_causal),
    "paged_causal": dict(layout_q="TND", layout_kv="PA_BBND", B=2, N1=2, N2=1, D=32,
                         lens_q=[300, 90], lens_kv=[300, 129], page_size=128, pattern=pat_random_k),
}


@pytest.mark.parametrize("name", sorted(CAUSAL_CASES))
def test_causal_sparse_equals_masked_dense(name):
    """Sparse + causal == dense attention under the selected-blocks-and-causal
    token mask; backward == autograd of the same."""
    p = make_problem(seed_base=zlib.crc32(name.encode()) % 983, causal=True, **CAUSAL_CASES[name])
    _compare_fwd(p)
    o = oracle.Oracle(p)
    out, lse, _ = o.fwd()
    dq, dk, dv, fl = o.bwd(out, p.dout, lse)
    rq, rk, rv = tr.grads(p, p.dout)
    assert fl == 0
    for a, r in ((dq, rq), (dk, rk), (dv, rv)):
        assert torch.allclose(a, r, atol=1e-10, rtol=0), (a - r).abs().max()


def test_causal_row_that_sees_nothing_is_empty():
    """A query block whose only selected kv block lies wholly after its rows
    sees no token under the mask: out 0, lse -inf (and zero gradients)."""
    def hook(rng, b, hi, i, sel):
        return [3] if i == 0 else sel
    p = make_problem(B=1, N1=1, N2=1, D=16, Sq=256, BQ=64, BKV=64, pattern=pat_causal,
                     row_hook=hook, seed_base=29, causal=True)
    o = oracle.Oracle(p)
    out, lse, fl = o.fwd()
    assert fl == 0
    assert torch.all(lse[0, 0, :64] == float("-inf")) and torch.all(out[0, 0, :64] == 0)
    assert torch.all(torch.isfinite(lse[0, 0, 64:]))
    dq, dk, dv, _ = o.bwd(out, p.dout, lse)
    assert torch.all(dq[0, 0, :64] == 0)


def test_causal_backward_finite_differences():
    """Central differences of L = sum(dOut * out) under the causal mask."""
    p = make_problem(layout_q="TND", layout_kv="TND", B=2, N1=2, N2=1, D=8, BQ=4, BKV=4,
                     lens_q=[9, 12], lens_kv=[14, 12], pattern=pat_random_k, seed_base=31,
                     dtype=torch.float64, causal=True)
    dout = p.dout.double()

    def loss(**kw):
        out, _, _ = oracle.Oracle(p, **kw).fwd()
        return float((out * dout).sum())

    o = oracle.Oracle(p)
    out, lse, _ = o.fwd()
    dq, dk, dv, _ = o.bwd(out, dout, lse)
    rng = np.random.default_rng(1)
    eps = 1e-6
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        base = getattr(p, name).double()
        for _ in range(6):
            pos = tuple(int(rng.integers(0, s)) for s in base.shape)
            plus, minus = base.clone(), base.clone()
            plus[pos] += eps
            minus[pos] -= eps
            args = {"q": p.q.double(), "k": p.k.double(), "v": p.v.double()}
            args[name] = plus
            lp = loss(**args)
            args[name] = minus
            lm = loss(**args)
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - float(grad[pos])) <= 1e-6 * max(1.0, abs(fd)), (name, pos, fd, float(grad[pos]))
