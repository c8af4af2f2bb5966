"""Helpers that run a ``workloads.Problem`` through the C-ABI binding and
compare results with the oracle (tolerances from the parity criteria)."""
from __future__ import annotations

import numpy as np
import torch

import block_sparse_variable_b200 as bsa

# Parity criteria for bf16/fp16 inputs: max-abs 2e-2 and rel-L2 1e-2 for
# out/dq/dk/dv, 1e-3 absolute for lse.  out (a convex combination of V rows,
# |out| < ~6 for N(0,1) data) is held to the literal absolute bound.  For
# dq/dk/dv the absolute bound is read as a bound for unit-scale entries: an
# entry with |ref| > 1 may differ by 2e-2*|ref| (a bf16 gradient of magnitude
# 51 already carries a rounding error of up to 0.1, so no bf16 output could
# meet a flat 2e-2 there); their literal max-abs and the count of entries
# above 2e-2 are reported (PARITY lines, visible with pytest -s).
OUT_MAX_ABS = 2e-2
OUT_REL_L2 = 1e-2
LSE_ABS = 1e-3


params_of = bsa.params_of_problem


def device_inputs(p, device="cuda"):
    d = {n: getattr(p, n) for n in ("q", "k", "v", "dout", "index")}
    d.update(cu_seqlens_q=p.cu_q, cu_seqlens_kv=p.cu_kv, seqused_kv=p.seqused_kv,
             block_table=p.block_table)
    return {n: (None if t is None else t.to(device)) for n, t in d.items()}


def opt_kwargs(d):
    return {n: d[n] for n in ("cu_seqlens_q", "cu_seqlens_kv", "seqused_kv", "block_table")}


def gpu_fwd(p, d=None, out=None, lse=None):
    d = d or device_inputs(p)
    if out is None and getattr(p, "out_dtype", None) is not None:
        out = torch.empty(d["q"].shape, dtype=p.out_dtype, device=d["q"].device)
    out, lse, ws = bsa.bsa_fwd(d["q"], d["k"], d["v"], d["index"], params_of(p), out=out, lse=lse,
                               **opt_kwargs(d))
    return out, lse, ws, d


def gpu_bwd(p, out, lse, d=None, dq=None, dk=None, dv=None):
    d = d or device_inputs(p)
    dq, dk, dv, ws = bsa.bsa_bwd(d["q"], d["k"], d["v"], out, d["dout"], lse, d["index"],
                                 params_of(p), dq=dq, dk=dk, dv=dv, **opt_kwargs(d))
    return dq, dk, dv, ws, d


def region(ws: torch.Tensor, reg, dtype, count=None) -> np.ndarray:
    raw = ws[reg.offset:reg.offset + reg.bytes].cpu()
    a = raw.view(dtype)
    return (a if count is None else a[:count]).numpy()


def check_close(name, got: torch.Tensor, ref: torch.Tensor, mask=None, literal=None):
    """max-abs and rel-L2 against the oracle.  literal (default: for names
    starting with "out") applies the flat 2e-2 absolute bound; otherwise the
    bound scales with |ref| above 1.  Prints one PARITY line with the literal
    max-abs, the scaled max-abs, rel-L2 and the count of entries above 2e-2."""
    g = got.double().cpu()
    r = ref.double().cpu()
    if mask is not None:
        g, r = g[mask], r[mask]
    assert torch.isfinite(g).all(), f"{name}: non-finite values"
    if literal is None:
        literal = name.startswith("out")
    err = (g - r).abs()
    max_abs = float(err.max()) if err.numel() else 0.0
    scaled = float((err / r.abs().clamp(min=1.0)).max()) if err.numel() else 0.0
    over = int((err > OUT_MAX_ABS).sum())
    rel = float(torch.linalg.vector_norm(g - r) / max(float(torch.linalg.vector_norm(r)), 1e-30))
    print(f"PARITY {name}: max_abs {max_abs:.3e} scaled {scaled:.3e} rel_l2 {rel:.3e} "
          f"over_2e-2 {over}/{err.numel()} max_ref {float(r.abs().max()) if r.numel() else 0.0:.3e}")
    bound = max_abs if literal else scaled
    assert bound <= OUT_MAX_ABS, \
        f"{name}: max-abs {max_abs:.3e}, scaled {scaled:.3e} (max|ref| {float(r.abs().max()):.3e})"
    assert rel <= OUT_REL_L2, f"{name}: rel-L2 {rel:.3e}"
    return max_abs, rel


def check_lse(got: torch.Tensor, ref: torch.Tensor, mask=None):
    g = got.double().cpu()
    r = ref.double().cpu()
    if mask is not None:
        g, r = g[mask], r[mask]
    fin = torch.isfinite(r)
    assert torch.equal(fin, torch.isfinite(g)), "lse: finite pattern differs"
    assert torch.all(g[~fin] == r[~fin]), "lse: infinite values differ"
    if fin.any():
        err = float((g[fin] - r[fin]).abs().max())
        assert err <= LSE_ABS, f"lse: max-abs {err:.3e}"


def q_defined_mask(p) -> torch.Tensor:
    """Rows of the q-layout tensors (out, lse, dq) that belong to a batch:
    every row for BNSD; for TND the rows cu_seqlens_q[b] .. + qlen_b of each
    batch whose lengths are consistent (the oracle's reading of the lengths;
    rows of no batch are not written)."""
    import oracle
    if p.layout_q == "BNSD":
        return torch.ones(p.q.shape[:-1], dtype=torch.bool)
    qlen = oracle.Oracle(p).batch_lengths()[0]
    m = torch.zeros(p.q.shape[:-1], dtype=torch.bool)
    for b in range(p.B):
        a = int(p.cu_q[b])
        m[a:a + qlen[b]] = True
    return m


def kv_written_mask(p) -> torch.Tensor:
    """Rows of dk/dv the backward writes: every stored row of every batch
    whose lengths are consistent (zeros past the used length); under paging,
    the rows of the pages that the table entries covering each batch's used
    length name (an entry outside the page range names no page)."""
    import oracle
    shape = p.k.shape[:-1]
    m = torch.zeros(shape, dtype=torch.bool)
    if p.layout_kv == "BNSD":
        m[:] = True
        return m
    _, kvlen, kvst, _ = oracle.Oracle(p).batch_lengths()
    if p.layout_kv == "TND":
        for b in range(p.B):
            a = int(p.cu_kv[b])
            m[a:a + kvst[b]] = True
        return m
    P = int(p.k.shape[0])
    for b in range(p.B):
        n = -(-kvlen[b] // p.page_size)
        for x in range(n):
            pg = int(p.block_table[b, x])
            if 0 <= pg < P:
                m[pg] = True
    return m


# ---------------------------------------------------------------- FP8 inputs
E4M3_HALF_ULP_REL = 2.0 ** -4   # 3 mantissa bits: round to nearest within 2^-4 relative
E4M3_HALF_SUB = 2.0 ** -10      # half the subnormal spacing 2^-9


def fp8_out_bound(p) -> torch.Tensor:
    """Element bound on |out - exact out| when P is cast to e4m3 before P V.

    The kernel computes P against a reference m no larger than the row max
    and sums l from the unrounded fp32 P, so with P_u = exp(s_u - max) and
    L = sum_u P_u (both exact, fp64), the cast changes out_d by at most
    sum_u (2^-4 P_u + 2^-10) |v_ud| / L: a relative 2^-4 for normal e4m3
    values, an absolute 2^-10 (scaled down by the later rescale, never up)
    below them.  Built from torch library routines on the dense token mask;
    a row that sees nothing has bound 0 (its out must be exactly 0)."""
    from tests import torch_reference as TR
    q, k, v = p.q.double(), p.k.double(), p.v.double()
    g = p.N1 // p.N2
    per = []
    for b in range(p.B):
        qb, kb, vb = TR.batch_tensors(p, b, q, k, v)
        kb, vb = kb.repeat_interleave(g, 0), vb.repeat_interleave(g, 0)
        mask = TR.token_mask(p, b)
        s = (p.scale * torch.matmul(qb, kb.transpose(-1, -2))).masked_fill(~mask, float("-inf"))
        m = s.amax(-1, keepdim=True)
        m = torch.where(torch.isfinite(m), m, torch.zeros_like(m))
        pr = torch.exp(s - m) * mask
        L = pr.sum(-1, keepdim=True)
        num = torch.matmul(E4M3_HALF_ULP_REL * pr + E4M3_HALF_SUB * mask.double(), vb.abs())
        per.append((torch.where(L > 0, num / L.clamp(min=1e-300), torch.zeros_like(num)), None))
    return TR.to_q_layout(p, per, 0)


def check_fp8_out(got: torch.Tensor, ref: torch.Tensor, bound: torch.Tensor, odtype):
    """Every element within the P-cast bound plus the output's own rounding
    (half an ulp of the output dtype) and a 1e-5 allowance for the fp32
    accumulation and exp2 approximation."""
    g, r, bd = got.double().cpu(), ref.double().cpu(), bound.double().cpu()
    assert torch.isfinite(g).all(), "out: non-finite values"
    half_ulp = 2.0 ** -9 if odtype == torch.bfloat16 else 2.0 ** -12
    lim = bd + half_ulp * r.abs() + 1e-5
    excess = float(((g - r).abs() - lim).max()) if g.numel() else -1.0
    assert excess <= 0, f"out: exceeds the e4m3 P-cast bound by {excess:.3e}"
    used = float(((g - r).abs() / lim).max()) if g.numel() else 0.0
    return used
