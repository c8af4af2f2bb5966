"""Helpers that run a ``workloads.Problem`` through the C-ABI binding and
compare results with the oracle (tolerances from the parity criteria)."""
from __future__ import annotations

import numpy as np
import torch

import block_sparse_variable_b200 as bsa

# Parity criteria for bf16/fp16 inputs: max-abs 2e-2 and rel-L2 1e-2 for
# out/dq/dk/dv, 1e-3 absolute for lse.  The absolute bound is read as a bound
# for unit-scale entries: an entry with |ref| > 1 may differ by 2e-2*|ref|
# (a bf16 result of magnitude 51 already carries a rounding error of up to
# 0.1, so no bf16 output could meet a flat 2e-2 there).
OUT_MAX_ABS = 2e-2
OUT_REL_L2 = 1e-2
LSE_ABS = 1e-3


def params_of(p, return_lse=True) -> bsa.Params:
    return bsa.params_for(p.layout_q, p.layout_kv, p.N1, p.N2, (p.BQ, p.BKV), p.scale, return_lse,
                          getattr(p, "causal", False), getattr(p, "deterministic", False))


def device_inputs(p, device="cuda"):
    d = {n: getattr(p, n) for n in ("q", "k", "v", "dout", "index")}
    d.update(cu_seqlens_q=p.cu_q, cu_seqlens_kv=p.cu_kv, seqused_kv=p.seqused_kv,
             block_table=p.block_table)
    return {n: (None if t is None else t.to(device)) for n, t in d.items()}


def opt_kwargs(d):
    return {n: d[n] for n in ("cu_seqlens_q", "cu_seqlens_kv", "seqused_kv", "block_table")}


def gpu_fwd(p, d=None, out=None, lse=None):
    d = d or device_inputs(p)
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


def check_close(name, got: torch.Tensor, ref: torch.Tensor, mask=None):
    g = got.double().cpu()
    r = ref.double().cpu()
    if mask is not None:
        g, r = g[mask], r[mask]
    assert torch.isfinite(g).all(), f"{name}: non-finite values"
    err = (g - r).abs()
    max_abs = float(err.max()) if err.numel() else 0.0
    scaled = float((err / r.abs().clamp(min=1.0)).max()) if err.numel() else 0.0
    rel = float(torch.linalg.vector_norm(g - r) / max(float(torch.linalg.vector_norm(r)), 1e-30))
    assert scaled <= OUT_MAX_ABS, \
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


def kv_written_mask(p) -> torch.Tensor:
    """Rows of dk/dv the backward writes (every stored row of every batch;
    under paging, the rows of the pages covering each batch's used length)."""
    shape = p.k.shape[:-1]
    if p.layout_kv != "PA_BBND":
        m = torch.zeros(shape, dtype=torch.bool)
        if p.layout_kv == "BNSD":
            m[:] = True
        else:
            m[:int(p.cu_kv[-1])] = True
        return m
    m = torch.zeros(shape, dtype=torch.bool)
    lens = p.seqused_kv.tolist()
    for b in range(p.B):
        n = -(-lens[b] // p.page_size)
        for x in range(n):
            m[int(p.block_table[b, x])] = True
    return m
