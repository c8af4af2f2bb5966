"""FP8 (e4m3) inputs: the pins of the oracle's input decode and of the
tolerance the GPU path is held to.

GenericBlockSparseAttention article, quantization table, quantType 5: q, k
and v are FLOAT8_E4M3 with no scale tensors, and P is cast to fp8 inside the
operator before the P V product; out is fp16 or bf16.  The oracle computes
the plain definition on the decoded inputs (no cast of P); the GPU result is
held to a bound derived from the e4m3 rounding of P (tests/harness.py,
fp8_out_bound)."""
import math

import numpy as np
import torch

import oracle
from tests import harness as H
from tests import torch_reference as TR
from workloads.gen import make_problem, pat_dense, pat_random_k


def _e4m3_by_definition(code: int) -> float:
    """OCP 8-bit floating point, E4M3: 1 sign, 4 exponent (bias 7), 3
    mantissa bits; exponent 0 is subnormal (2^-6 * m/8); S.1111.111 is NaN
    and there is no infinity."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return s * 2.0 ** -6 * (m / 8.0)
    return s * 2.0 ** (e - 7) * (1.0 + m / 8.0)


def test_e4m3_decode_is_the_format_definition():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    lib = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ref = np.array([_e4m3_by_definition(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(lib))
    assert np.array_equal(ref[~nan], lib[~nan])
    assert ref[~nan].max() == 448.0 and ref[1] == 2.0 ** -9


def test_fp8_inputs_reach_the_oracle_exactly():
    """The oracle's dense result on e4m3 inputs is torch's fp64 softmax
    attention on the same decoded values."""
    p = make_problem(layout_q="BNSD", layout_kv="BNSD", B=1, N1=2, N2=1, D=128, Sq=200,
                     dtype=torch.float8_e4m3fn, pattern=pat_dense, seed_base=31)
    out, lse, fl = oracle.Oracle(p).fwd()
    assert fl == 0 and out.dtype == torch.float64
    q, k, v = (t.double() for t in (p.q, p.k, p.v))
    k, v = k.repeat_interleave(2, 1), v.repeat_interleave(2, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=p.scale)
    assert float((out - ref).abs().max()) < 1e-12
    ref_lse = torch.logsumexp(p.scale * q @ k.transpose(-1, -2), -1)
    assert float((lse - ref_lse).abs().max()) < 1e-12


def _cast_model(p):
    """P cast to e4m3 in the row-max scale (torch's own fp32 -> e4m3
    conversion, round to nearest even, saturating), l from the unrounded P."""
    q, k, v = p.q.double(), p.k.double(), p.v.double()
    g = p.N1 // p.N2
    per = []
    for b in range(p.B):
        qb, kb, vb = TR.batch_tensors(p, b, q, k, v)
        kb, vb = kb.repeat_interleave(g, 0), vb.repeat_interleave(g, 0)
        mask = TR.token_mask(p, b)
        s = (p.scale * qb @ kb.transpose(-1, -2)).masked_fill(~mask, float("-inf"))
        m = s.amax(-1, keepdim=True)
        pr = torch.exp(s - m).nan_to_num(0.0)
        pq = pr.float().to(torch.float8_e4m3fn).double()
        per.append((pq @ vb / pr.sum(-1, keepdim=True), None))
    return TR.to_q_layout(p, per, 0)


def test_the_bound_covers_a_model_of_the_cast():
    """The bound holds for P cast in the row-max scale, and is not vacuous:
    the cast model's error uses a visible part of it."""
    for seed, pat in ((41, pat_dense), (43, pat_random_k)):
        p = make_problem(layout_q="TND", layout_kv="TND", B=2, N1=2, N2=2, D=128,
                         lens_q=[260, 130], lens_kv=[300, 200], dtype=torch.float8_e4m3fn,
                         pattern=pat, seed_base=seed)
        exact, _, _ = oracle.Oracle(p).fwd()
        model = _cast_model(p)
        bound = H.fp8_out_bound(p)
        err = (model - exact).abs()
        assert bool((err <= bound + 1e-12).all())
        assert float((err / bound.clamp(min=1e-30)).max()) > 0.05
