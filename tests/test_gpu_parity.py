"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs.  Builders (compacted rows, inverse index, work lists,
status flags) must match exactly; out/dq/dk/dv within max-abs 2e-2 and
rel-L2 1e-2; lse within 1e-3.  Backward inputs are the oracle's out rounded
to the input dtype and its lse in fp32, given to both sides."""
import math
import zlib

import numpy as np
import pytest
import torch

import block_sparse_variable_b200 as bsa
import oracle
import workloads
from oracle import builders
from workloads.gen import (make_problem, pat_dense, pat_density, pat_fraction_diag, pat_random_k,
                           pat_topk)
from tests import harness as H

pytestmark = pytest.mark.gpu

SMALL = {
    "bnsd_random": dict(layout_q="BNSD", layout_kv="BNSD", B=2, N1=2, N2=2, D=64, Sq=384,
                        pattern=pat_random_k),
    "bnsd_ragged_kv": dict(layout_q="BNSD", layout_kv="BNSD", B=2, N1=2, N2=1, D=64, Sq=300,
                           lens_kv=[300, 170], Skv=300, pattern=pat_density(0.5, 1)),
    "bnsd_blocks_256x128": dict(layout_q="BNSD", layout_kv="BNSD", B=1, N1=2, N2=2, D=128,
                                Sq=640, BQ=256, BKV=128, pattern=pat_density(0.4, 1)),
    "bnsd_fp16_d128": dict(layout_q="BNSD", layout_kv="BNSD", B=1, N1=3, N2=1, D=128, Sq=520,
                           dtype=torch.float16, pattern=pat_random_k),
    "tnd_gqa": dict(layout_q="TND", layout_kv="TND", B=3, N1=4, N2=2, D=64,
                    lens_q=[130, 300, 77], lens_kv=[200, 129, 256], pattern=pat_fraction_diag(0.5)),
    "tnd_gqa_d128": dict(layout_q="TND", layout_kv="TND", B=2, N1=8, N2=2, D=128,
                         lens_q=[600, 257], lens_kv=[600, 257], pattern=pat_fraction_diag(0.25)),
    "tnd_shared_rows": dict(layout_q="TND", layout_kv="TND", B=2, N1=4, N2=2, Hidx=2, D=64,
                            lens_q=[256, 140], lens_kv=[256, 140], pattern=pat_random_k),
    "tnd_seqused": dict(layout_q="TND", layout_kv="TND", B=2, N1=2, N2=2, D=64,
                        lens_q=[200, 90], lens_kv=[150, 60], kv_storage=[260, 100],
                        pattern=pat_random_k),
    "tnd_empty_batches": dict(layout_q="TND", layout_kv="TND", B=3, N1=2, N2=2, D=64,
                              lens_q=[0, 150, 40], lens_kv=[100, 0, 300], pattern=pat_random_k),
    "paged": dict(layout_q="TND", layout_kv="PA_BBND", B=3, N1=4, N2=2, D=64,
                  lens_q=[300, 129, 64], lens_kv=[300, 129, 64], page_size=128, extra_pages=2,
                  pattern=pat_topk(2)),
    "paged_256": dict(layout_q="TND", layout_kv="PA_BBND", B=2, N1=2, N2=1, D=128,
                      lens_q=[700, 130], lens_kv=[600, 300], page_size=256, extra_pages=1,
                      dtype=torch.float16, pattern=pat_random_k),
    "big_blocks": dict(layout_q="TND", layout_kv="TND", B=2, N1=2, N2=2, D=64, BQ=512, BKV=256,
                       lens_q=[700, 300], lens_kv=[900, 300], pattern=pat_random_k),
    "blocks_1024": dict(layout_q="BNSD", layout_kv="BNSD", B=1, N1=2, N2=2, D=64, Sq=1500,
                        BQ=1024, BKV=1024, dtype=torch.float16, pattern=pat_random_k),
    "dense_many_blocks": dict(layout_q="BNSD", layout_kv="BNSD", B=1, N1=1, N2=1, D=128, Sq=1100,
                              pattern=pat_dense),
}


def _hook_invalid(rng, b, hi, i, sel):
    if i == 0 and hi == 0:
        return [1, 0xFFFF, 1, 0, 3, 9]
    return sel


def _hook_empty(rng, b, hi, i, sel):
    return [] if (i % 2 == 1) else sel


EDGE = {
    "invalid_entries": dict(layout_q="BNSD", layout_kv="BNSD", B=1, N1=2, N2=2, D=64, Sq=512, W=6,
                            pattern=pat_random_k, row_hook=_hook_invalid),
    "empty_rows": dict(layout_q="TND", layout_kv="TND", B=2, N1=2, N2=1, D=64,
                       lens_q=[384, 200], lens_kv=[256, 300], pattern=pat_random_k,
                       row_hook=_hook_empty),
}


# causal mask aligned to the end of the kv sequence: query row t sees kv
# token u iff u <= t + kvlen - qlen (rows with nothing visible: lse -inf, out 0)
CAUSAL = {
    "causal_bnsd_dense": dict(layout_q="BNSD", layout_kv="BNSD", B=1, N1=2, N2=2, D=128, Sq=640,
                              pattern=pat_dense, causal=True),
    "causal_bnsd_128x512": dict(layout_q="BNSD", layout_kv="BNSD", B=2, N1=2, N2=1, D=64, Sq=1100,
                                BKV=512, pattern=pat_dense, causal=True),
    "causal_bnsd_ragged_kv": dict(layout_q="BNSD", layout_kv="BNSD", B=2, N1=2, N2=2, D=64, Sq=300,
                                  lens_kv=[300, 470], Skv=470, pattern=pat_dense, causal=True),
    "causal_tnd_gqa_prefix": dict(layout_q="TND", layout_kv="TND", B=3, N1=4, N2=2, D=64,
                                  lens_q=[130, 300, 77], lens_kv=[400, 300, 205],
                                  pattern=pat_random_k, causal=True),
    "causal_tnd_q_longer": dict(layout_q="TND", layout_kv="TND", B=2, N1=2, N2=1, D=128,
                                lens_q=[300, 140], lens_kv=[150, 140], pattern=pat_dense,
                                causal=True),
    "causal_tnd_fp16_256x256": dict(layout_q="TND", layout_kv="TND", B=2, N1=2, N2=2, D=128,
                                    BQ=256, BKV=256, lens_q=[700, 260], lens_kv=[700, 500],
                                    dtype=torch.float16, pattern=pat_density(0.7, 1), causal=True),
    "causal_paged": dict(layout_q="TND", layout_kv="PA_BBND", B=3, N1=4, N2=2, D=64,
                         lens_q=[200, 129, 64], lens_kv=[456, 129, 300], page_size=128,
                         extra_pages=2, pattern=pat_dense, causal=True),
}


def _problem(name):
    spec = dict(SMALL.get(name) or EDGE.get(name) or CAUSAL[name])
    return make_problem(seed_base=zlib.crc32(name.encode()) % 9973, name=name, **spec)


def _oracle(p):
    o = oracle.Oracle(p)
    out, lse, fl = o.fwd()
    out_b = out.to(p.dtype)
    lse_f = lse.float()
    dq, dk, dv, fl2 = o.bwd(out_b, p.dout, lse_f)
    return dict(out=out, lse=lse, out_b=out_b, lse_f=lse_f, dq=dq, dk=dk, dv=dv,
                flags=fl | fl2 | o.scan_flags())


def _check_builders(p, ws_f, ws_b, lay_f, lay_b, B):
    st_f = H.region(ws_f, lay_f.status, torch.int32).astype(np.int64)
    st_b = H.region(ws_b, lay_b.status, torch.int32).astype(np.int64)
    geo = B["geo"]
    assert st_f[0] == B["flags"] and st_b[0] == B["flags"]
    assert st_f[5] == geo.TK and st_b[5] == geo.TK
    n_f = int(st_f[2])
    assert n_f == len(B["fwd_items"])
    Hidx, Rg, W = p.Hidx, geo.Rg, p.W
    comp = H.region(ws_f, lay_f.comp, torch.int16).view(np.uint16).reshape(Hidx, Rg, W)
    ncomp = H.region(ws_f, lay_f.ncomp, torch.int32).reshape(Hidx, Rg)
    assert np.array_equal(ncomp, B["ncomp"])
    assert np.array_equal(comp, B["comp"])
    assert np.array_equal(H.region(ws_f, lay_f.fwd_items, torch.int32, n_f), B["fwd_items"])
    nnz = int(st_b[6])
    off = H.region(ws_b, lay_b.inv_off, torch.int32, Hidx * geo.TK + 1)
    assert np.array_equal(off, B["inv_off"]) and nnz == len(B["inv_list"])
    assert np.array_equal(H.region(ws_b, lay_b.inv_list, torch.int32, nnz), B["inv_list"])
    n_b = int(st_b[4])
    assert n_b == len(B["bwd_items"])
    assert np.array_equal(H.region(ws_b, lay_b.bwd_items, torch.int32, n_b), B["bwd_items"])


def _run_and_check(p):
    R = _oracle(p)
    Bld = builders.build_all(p)
    d = H.device_inputs(p)
    # sentinel-filled outputs: rows that belong to no batch must stay untouched
    out0 = torch.full(d["q"].shape, float("nan"), dtype=p.odtype, device="cuda")
    lse0 = torch.full(oracle.Oracle(p).lse_shape(), float("nan"), dtype=torch.float32,
                      device="cuda")
    out, lse, ws_f, _ = H.gpu_fwd(p, d, out=out0, lse=lse0)
    torch.cuda.synchronize()
    qmask = H.q_defined_mask(p)
    H.check_close("out", out, R["out"], qmask)
    H.check_lse(lse, R["lse"], qmask)
    if (~qmask).any():
        assert torch.isnan(out.cpu()[~qmask].float()).all() and torch.isnan(lse.cpu()[~qmask]).all()
    # backward on the oracle's (rounded) forward results; sentinel-filled outputs
    dk0 = torch.full_like(d["k"], float("nan"))
    dv0 = torch.full_like(d["v"], float("nan"))
    dq0 = torch.full_like(d["q"], float("nan"))
    dq, dk, dv, ws_b, _ = H.gpu_bwd(p, R["out_b"].cuda(), R["lse_f"].cuda(), d, dq=dq0, dk=dk0, dv=dv0)
    torch.cuda.synchronize()
    wm = H.kv_written_mask(p)
    H.check_close("dq", dq, R["dq"], qmask)
    H.check_close("dk", dk, R["dk"], wm)
    H.check_close("dv", dv, R["dv"], wm)
    if (~wm).any():   # rows the backward must leave alone stay untouched
        assert torch.isnan(dk.cpu()[~wm]).all() and torch.isnan(dv.cpu()[~wm]).all()
    lay_f = bsa.bsa_fwd_workspace_layout(d["q"], d["k"], d["v"], d["index"], H.params_of(p),
                                         lse=lse, **H.opt_kwargs(d))
    lay_b = bsa.bsa_bwd_workspace_layout(d["q"], d["k"], d["v"], out, d["dout"], lse, d["index"],
                                         H.params_of(p), **H.opt_kwargs(d))
    _check_builders(p, ws_f, ws_b, lay_f, lay_b, Bld)
    assert bsa.bsa_read_status(ws_f) == R["flags"]


# Data values that contradict the tensors they describe (GenericBlockSparse-
# Attention article: values are not checked at tiling; the dual-length rule
# for seqused_kv; paged addressing), the readings pinned on the oracle by
# tests/test_corrupt_inputs.py: a contradictory length counts as 0
# (BAD_SEQLEN), a table entry outside the page range drops the tokens it
# covers (BAD_PAGE, raised whether or not a row selects them), a query block
# without an index row selects nothing (BAD_INDEX).  No fault, no write to a
# row of no batch, outputs and the flag word equal to the oracle's.
def _corrupt(name):
    seed = zlib.crc32(name.encode()) % 9973
    if name == "tnd_q_batches_out_of_order":
        # batch 1's cu_seqlens_q pair decreases; batches 0 and 2 swap places
        p = make_problem(seed_base=seed, name=name, layout_q="TND", layout_kv="TND", B=3, N1=4,
                         N2=2, D=64, lens_q=[300, 0, 200], lens_kv=[260, 140, 330],
                         pattern=pat_random_k)
        p.cu_q = torch.tensor([200, 500, 0, 200], dtype=torch.int64)
    elif name == "tnd_q_past_end":
        p = make_problem(seed_base=seed, name=name, layout_q="TND", layout_kv="TND", B=2, N1=2,
                         N2=1, D=128, lens_q=[200, 150], lens_kv=[200, 330], pattern=pat_random_k)
        p.cu_q = torch.tensor([0, 200, 360], dtype=torch.int64)   # 360 > Tq = 350
    elif name == "tnd_kv_past_end":
        p = make_problem(seed_base=seed, name=name, layout_q="TND", layout_kv="TND", B=2, N1=2,
                         N2=2, D=64, lens_q=[200, 150], lens_kv=[300, 180], pattern=pat_random_k)
        p.cu_kv = torch.tensor([0, 300, 680], dtype=torch.int64)  # 680 > Tkv = 480
    elif name == "tnd_seqused_over_storage":
        p = make_problem(seed_base=seed, name=name, layout_q="TND", layout_kv="TND", B=2, N1=2,
                         N2=2, D=64, lens_q=[200, 90], lens_kv=[150, 60], kv_storage=[260, 100],
                         pattern=pat_random_k)
        p.seqused_kv = torch.tensor([150, 101], dtype=torch.int32)  # 101 > 100 stored
    elif name == "paged_bad_table_entries":
        p = make_problem(seed_base=seed, name=name, layout_q="TND", layout_kv="PA_BBND", B=3,
                         N1=4, N2=2, D=64, lens_q=[300, 129, 64], lens_kv=[300, 129, 300],
                         page_size=128, extra_pages=2, pattern=pat_random_k)
        bt = p.block_table.clone()
        P = int(p.k.shape[0])
        bt[0, 1] = -1          # inside batch 0's used length
        bt[2, 0] = P + 5       # inside batch 2's used length
        bt[1, 2] = -7          # past batch 1's used length: no flag
        p.block_table = bt
    elif name == "tnd_index_too_few_rows":
        p = make_problem(seed_base=seed, name=name, layout_q="TND", layout_kv="TND", B=2, N1=2,
                         N2=1, D=64, lens_q=[300, 260], lens_kv=[300, 400], pattern=pat_random_k)
        p.index = p.index[:, :4].contiguous()   # the lengths need 3 + 3 rows
    elif name == "bnsd_seqused_negative":
        p = make_problem(seed_base=seed, name=name, layout_q="BNSD", layout_kv="BNSD", B=2, N1=2,
                         N2=1, D=64, Sq=256, lens_kv=[256, 200], Skv=256, pattern=pat_random_k)
        p.seqused_kv = torch.tensor([-3, 200], dtype=torch.int32)
    else:
        raise KeyError(name)
    return p


CORRUPT = ["tnd_q_batches_out_of_order", "tnd_q_past_end", "tnd_kv_past_end",
           "tnd_seqused_over_storage", "paged_bad_table_entries", "tnd_index_too_few_rows",
           "bnsd_seqused_negative"]


@pytest.mark.parametrize("name", CORRUPT)
def test_corrupt_lengths_pages_index(name):
    p = _corrupt(name)
    assert oracle.Oracle(p).scan_flags() != 0
    _run_and_check(p)


@pytest.mark.parametrize("name", ["tnd_q_batches_out_of_order", "paged_bad_table_entries",
                                  "tnd_index_too_few_rows"])
def test_corrupt_inputs_deterministic_backward(name):
    _check_deterministic(_corrupt(name))


# Packed GQA tiles (GenericBlockSparseAttention, attribute isPackedGQA): the g
# query heads of a group share their index row (Hidx == N2) and, for g in
# {2, 4, 8, 16}, the forward packs 128/g rows of each head into one tile.
# g = 3 shares the row but keeps one head per tile.
PACKED = {
    "packed_tnd_g4_d128": dict(layout_q="TND", layout_kv="TND", B=3, N1=16, N2=4, Hidx=4, D=128,
                               lens_q=[300, 130, 517], lens_kv=[300, 700, 517],
                               pattern=pat_fraction_diag(0.3)),
    "packed_bnsd_g8": dict(layout_q="BNSD", layout_kv="BNSD", B=1, N1=8, N2=1, Hidx=1, D=64,
                           Sq=300, BKV=256, pattern=pat_random_k),
    "packed_bnsd_g16_bq256": dict(layout_q="BNSD", layout_kv="BNSD", B=2, N1=16, N2=1, Hidx=1,
                                  D=64, Sq=200, BQ=256, pattern=pat_random_k),
    "packed_paged_g4_fp16": dict(layout_q="TND", layout_kv="PA_BBND", B=3, N1=8, N2=2, Hidx=2,
                                 D=128, lens_q=[300, 129, 64], lens_kv=[300, 129, 64],
                                 page_size=128, extra_pages=2, dtype=torch.float16,
                                 pattern=pat_topk(2)),
    "packed_causal_g4": dict(layout_q="TND", layout_kv="TND", B=2, N1=8, N2=2, Hidx=2, D=64,
                             lens_q=[300, 140], lens_kv=[500, 140], pattern=pat_dense, causal=True),
    "packed_bq512_g2": dict(layout_q="TND", layout_kv="TND", B=2, N1=4, N2=2, Hidx=2, D=64,
                            BQ=512, BKV=256, lens_q=[700, 300], lens_kv=[900, 300],
                            pattern=pat_random_k),
    "shared_rows_g3_unpacked": dict(layout_q="TND", layout_kv="TND", B=2, N1=6, N2=2, Hidx=2,
                                    D=64, lens_q=[260, 140], lens_kv=[260, 300],
                                    pattern=pat_random_k),
}


def _packed_problem(name):
    return make_problem(seed_base=zlib.crc32(name.encode()) % 9973, name=name, **PACKED[name])


@pytest.mark.parametrize("name", sorted(PACKED))
def test_packed_gqa(name):
    p = _packed_problem(name)
    g = p.N1 // p.N2
    assert builders.packed_heads(p) == (g if g in (2, 4, 8, 16) else 1)
    _run_and_check(p)


@pytest.mark.parametrize("name", ["packed_tnd_g4_d128", "packed_paged_g4_fp16", "packed_causal_g4"])
def test_packed_gqa_equals_per_head_rows(name):
    """The same problem with the group's row copied to every head (Hidx ==
    N1, one head per tile) gives the same forward within rounding."""
    p = _packed_problem(name)
    g = p.N1 // p.N2
    d = H.device_inputs(p)
    out_p, lse_p, _, _ = H.gpu_fwd(p, d)
    hdim = 1 if p.layout_q == "BNSD" else 0
    p.index = p.index.view(torch.int16).repeat_interleave(g, dim=hdim).view(torch.uint16)
    p.Hidx = p.N1
    d = H.device_inputs(p)
    out_h, lse_h, _, _ = H.gpu_fwd(p, d)
    torch.cuda.synchronize()
    H.check_close("out(packed vs per-head)", out_p, out_h.double())
    H.check_lse(lse_p, lse_h)


@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_cases(name):
    _run_and_check(_problem(name))


@pytest.mark.parametrize("name", sorted(EDGE))
def test_edge_cases(name):
    _run_and_check(_problem(name))


@pytest.mark.parametrize("name", sorted(CAUSAL))
def test_causal_cases(name):
    p = _problem(name)
    assert p.causal
    _run_and_check(p)


# deterministic backward: dK/dV from the kv-major kernel without its dQ
# reductions, dQ from the q-major pass; parity as above, the forward work
# list in the backward workspace exact, and a second call bitwise identical
DETERMINISTIC = ["bnsd_random", "bnsd_ragged_kv", "bnsd_blocks_256x128", "bnsd_fp16_d128",
                 "tnd_gqa", "tnd_shared_rows", "tnd_seqused", "tnd_empty_batches", "paged",
                 "paged_256", "big_blocks", "blocks_1024", "dense_many_blocks", "invalid_entries",
                 "empty_rows", "causal_tnd_q_longer", "causal_paged", "causal_bnsd_128x512"]


def _check_deterministic(p):
    p.deterministic = True
    _run_and_check(p)
    R = _oracle(p)
    d = H.device_inputs(p)
    out_b, lse_f = R["out_b"].cuda(), R["lse_f"].cuda()
    first = H.gpu_bwd(p, out_b, lse_f, d)
    second = H.gpu_bwd(p, out_b, lse_f, d)
    torch.cuda.synchronize()
    wm = H.kv_written_mask(p).cuda()  # paged: pages the call does not own stay untouched
    qm = H.q_defined_mask(p).cuda()   # rows of no batch are not written
    for name, a, b in zip(("dq", "dk", "dv"), first[:3], second[:3]):
        a, b = (a[qm], b[qm]) if name == "dq" else (a[wm], b[wm])
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), f"{name} differs between runs"
    ws_b = first[3]
    lay_b = bsa.bsa_bwd_workspace_layout(d["q"], d["k"], d["v"], out_b, d["dout"], lse_f, d["index"],
                                         H.params_of(p), **H.opt_kwargs(d))
    assert lay_b.dq_acc.bytes == 0 and lay_b.fwd_items.bytes > 0
    st = H.region(ws_b, lay_b.status, torch.int32)
    B = builders.build_all(p)
    n_f = int(st[2])
    # the q-major pass takes one head per item, packed or not
    assert n_f == len(B["fwd_items_per_head"])
    assert np.array_equal(H.region(ws_b, lay_b.fwd_items, torch.int32, n_f), B["fwd_items_per_head"])


@pytest.mark.parametrize("name", DETERMINISTIC)
def test_deterministic_backward(name):
    _check_deterministic(_problem(name))


@pytest.mark.parametrize("name", ["tnd_seqused", "paged_256"])
def test_deterministic_backward_nan_in_unused_kv(name):
    _check_deterministic(_poison_unused_kv(_problem(name)))


@pytest.mark.parametrize("c", [1, 2])
def test_deterministic_backward_configs(c):
    _check_deterministic(workloads.make_config(c))


def _poison_unused_kv(p):
    """NaN in every stored K/V row the attention must not use: rows past
    seqused_kv (BNSD, TND), the tail of each last page and whole unused pages
    (PA_BBND).  Results must not change and must stay finite."""
    k, v = p.k.clone(), p.v.clone()
    lens = p.lens_kv
    if p.layout_kv == "BNSD":
        for b, n in enumerate(lens):
            k[b, :, n:] = float("nan")
            v[b, :, n:] = float("nan")
    elif p.layout_kv == "TND":
        cu = p.cu_kv.tolist()
        for b, n in enumerate(lens):
            k[cu[b] + n:cu[b + 1]] = float("nan")
            v[cu[b] + n:cu[b + 1]] = float("nan")
    else:
        used = set()
        ps = p.page_size
        for b, n in enumerate(lens):
            for j in range((n + ps - 1) // ps):
                pg = int(p.block_table[b, j])
                used.add(pg)
                if (j + 1) * ps > n:
                    k[pg, n - j * ps:] = float("nan")
                    v[pg, n - j * ps:] = float("nan")
        for pg in range(k.shape[0]):
            if pg not in used:
                k[pg] = float("nan")
                v[pg] = float("nan")
    p.k, p.v = k, v
    return p


@pytest.mark.parametrize("name", ["bnsd_ragged_kv", "tnd_seqused", "paged", "paged_256"])
def test_nan_in_unused_kv_rows(name):
    p = _poison_unused_kv(_problem(name))
    assert torch.isnan(p.k.float()).any()
    _run_and_check(p)


@pytest.mark.parametrize("c", [1, 2])
def test_configs_full(c):
    _run_and_check(workloads.make_config(c))


def test_return_lse_off_and_repeat_calls():
    """lse may be omitted; a reused workspace gives identical results."""
    p = _problem("tnd_gqa")
    d = H.device_inputs(p)
    P = H.params_of(p, return_lse=False)
    out1, lse1, ws = bsa.bsa_fwd(d["q"], d["k"], d["v"], d["index"], P, **H.opt_kwargs(d))
    assert lse1 is None
    out2, _, _ = bsa.bsa_fwd(d["q"], d["k"], d["v"], d["index"], P, workspace=ws, **H.opt_kwargs(d))
    torch.cuda.synchronize()
    assert torch.equal(out1, out2)


def test_chain_gpu_forward_then_backward():
    """GPU fwd -> GPU bwd against oracle fwd -> oracle bwd."""
    p = _problem("tnd_gqa_d128")
    o = oracle.Oracle(p)
    out, lse, _ = o.fwd()
    dq, dk, dv, _ = o.bwd(out, p.dout, lse)
    g_out, g_lse, _, d = H.gpu_fwd(p)
    g_dq, g_dk, g_dv, _, _ = H.gpu_bwd(p, g_out, g_lse, d)
    torch.cuda.synchronize()
    H.check_close("dq", g_dq, dq)
    H.check_close("dk", g_dk, dk)
    H.check_close("dv", g_dv, dv)


# --------------------------------------------------------------- full sizes
def _heads_of(o, rows, heads):
    """Rows (b, h1, t) whose (batch, head) -- BNSD -- or head -- TND -- is in heads."""
    p = o.prob
    keys = rows[:, 0] * p.N1 + rows[:, 1] if p.layout_q == "BNSD" else rows[:, 1]
    return rows[np.isin(keys, heads)]


@pytest.mark.parametrize("c", [3, 4, 5])
def test_configs_full_size_sampled(c):
    """Full-size workloads, launched exactly as the benchmark does: builders
    compared in full; the forward on every row of 4 seeded heads (BNSD: 4
    (batch, head) pairs); the backward on one whole kv-head group -- every
    dk/dv row of the group and every dq row of its query heads.  The
    backward's out/lse come from the oracle for the group's heads; other
    heads get out 0 and lse +inf, so they add nothing."""
    p = workloads.make_config(c)
    o = oracle.Oracle(p)
    rng = np.random.default_rng(c)
    d = H.device_inputs(p)
    out, lse, ws_f, _ = H.gpu_fwd(p, d)
    torch.cuda.synchronize()
    all_rows = o.q_rows_all()
    nheads = p.B * p.N1 if p.layout_q == "BNSD" else p.N1
    heads = rng.choice(nheads, size=4, replace=False)
    rows = _heads_of(o, all_rows, heads)
    r_out, r_lse, fl = o.fwd_rows(rows)
    H.check_close(f"out(C{c}, 4 heads, {len(rows)} rows)", o.gather_q(out.cpu(), rows),
                  torch.from_numpy(r_out))
    H.check_lse(o.gather_q(lse.cpu(), rows), torch.from_numpy(r_lse))

    # builders in full
    Bld = builders.build_all(p)
    lay_f = bsa.bsa_fwd_workspace_layout(d["q"], d["k"], d["v"], d["index"], H.params_of(p),
                                         lse=lse, **H.opt_kwargs(d))
    st = H.region(ws_f, lay_f.status, torch.int32)
    assert st[0] == Bld["flags"] == 0
    n_f = int(st[2])
    assert np.array_equal(H.region(ws_f, lay_f.fwd_items, torch.int32, n_f), Bld["fwd_items"])

    # backward on the kv-head group of the first sampled head
    g = p.N1 // p.N2
    if p.layout_q == "BNSD":
        b_sel, h2 = int(heads[0]) // p.N1, (int(heads[0]) % p.N1) // g
        grp = (all_rows[:, 0] == b_sel) & (all_rows[:, 1] // g == h2)
    else:
        b_sel, h2 = None, int(heads[0]) // g
        grp = all_rows[:, 1] // g == h2
    grows = all_rows[grp]
    g_out, g_lse, _ = o.fwd_rows(grows)
    out_in = torch.zeros(p.q.shape, dtype=p.dtype)
    lse_in = torch.full(o.lse_shape(), float("inf"), dtype=torch.float32)
    o._scatter_q(out_in, grows, torch.from_numpy(g_out).to(p.dtype))
    o._scatter_stat(lse_in, grows, torch.from_numpy(g_lse).float())
    dq, dk, dv, ws_b, _ = H.gpu_bwd(p, out_in.cuda(), lse_in.cuda(), d)
    torch.cuda.synchronize()
    r_dq, _ = o.bwd_dq_rows(out_in, p.dout, lse_in, grows)
    H.check_close(f"dq(C{c}, group, {len(grows)} rows)", o.gather_q(dq.cpu(), grows),
                  torch.from_numpy(r_dq))
    kvr = o.kv_rows_all()
    kvr = kvr[kvr[:, 1] == h2]
    if b_sel is not None:
        kvr = kvr[kvr[:, 0] == b_sel]
    r_dk, r_dv, _ = o.bwd_dkv_rows(out_in, p.dout, lse_in, kvr)
    ix = o.kv_index(kvr)
    H.check_close(f"dk(C{c}, group, {len(kvr)} rows)", dk.cpu()[ix], torch.from_numpy(r_dk))
    H.check_close(f"dv(C{c}, group, {len(kvr)} rows)", dv.cpu()[ix], torch.from_numpy(r_dv))
    lay_b = bsa.bsa_bwd_workspace_layout(d["q"], d["k"], d["v"], out, d["dout"], lse, d["index"],
                                         H.params_of(p), **H.opt_kwargs(d))
    stb = H.region(ws_b, lay_b.status, torch.int32)
    assert stb[4] == len(Bld["bwd_items"])
    assert np.array_equal(H.region(ws_b, lay_b.bwd_items, torch.int32, int(stb[4])), Bld["bwd_items"])
    nnz = int(stb[6])
    assert np.array_equal(H.region(ws_b, lay_b.inv_list, torch.int32, nnz), Bld["inv_list"])


# ------------------------------------------------------------- FP8 forward
# q, k, v in e4m3, P cast to e4m3 before P V (GenericBlockSparseAttention,
# quantization table, quantType 5); out within the P-cast bound of the exact
# oracle (tests/harness.py, fp8_out_bound), lse within 1e-3
FP8 = {
    "fp8_bnsd_dense": dict(layout_q="BNSD", layout_kv="BNSD", B=1, N1=2, N2=2, D=128, Sq=640,
                           pattern=pat_dense),
    "fp8_bnsd_ragged_kv": dict(layout_q="BNSD", layout_kv="BNSD", B=2, N1=2, N2=1, D=128, Sq=300,
                               lens_kv=[300, 170], Skv=300, pattern=pat_density(0.6, 1)),
    "fp8_tnd_gqa_fp16_out": dict(layout_q="TND", layout_kv="TND", B=3, N1=4, N2=2, D=128,
                                 lens_q=[130, 300, 77], lens_kv=[200, 129, 256],
                                 out_dtype=torch.float16, pattern=pat_random_k),
    "fp8_paged": dict(layout_q="TND", layout_kv="PA_BBND", B=2, N1=4, N2=2, D=128,
                      lens_q=[300, 129], lens_kv=[456, 129], page_size=128, extra_pages=2,
                      pattern=pat_topk(2)),
    "fp8_big_blocks": dict(layout_q="TND", layout_kv="TND", B=2, N1=2, N2=2, D=128, BQ=256,
                           BKV=512, lens_q=[700, 300], lens_kv=[900, 300], pattern=pat_random_k),
    "fp8_causal": dict(layout_q="TND", layout_kv="TND", B=2, N1=2, N2=1, D=128,
                       lens_q=[300, 140], lens_kv=[500, 140], pattern=pat_dense, causal=True),
    "fp8_empty_rows": dict(layout_q="TND", layout_kv="TND", B=2, N1=2, N2=1, D=128,
                           lens_q=[384, 200], lens_kv=[256, 300], pattern=pat_random_k,
                           row_hook=_hook_empty),
    "fp8_packed_g4": dict(layout_q="TND", layout_kv="TND", B=2, N1=8, N2=2, Hidx=2, D=128,
                          lens_q=[300, 140], lens_kv=[400, 140], pattern=pat_random_k),
}


def _fp8_problem(name):
    return make_problem(seed_base=zlib.crc32(name.encode()) % 9973, name=name,
                        dtype=torch.float8_e4m3fn, **FP8[name])


def _check_fp8(p):
    out_ref, lse_ref, fl = oracle.Oracle(p).fwd()
    d = H.device_inputs(p)
    out, lse, ws, _ = H.gpu_fwd(p, d)
    torch.cuda.synchronize()
    assert out.dtype == p.odtype
    H.check_fp8_out(out, out_ref, H.fp8_out_bound(p), p.odtype)
    H.check_lse(lse, lse_ref)
    assert bsa.bsa_read_status(ws) == (fl | oracle.Oracle(p).scan_flags())


@pytest.mark.parametrize("name", sorted(FP8))
def test_fp8_forward(name):
    _check_fp8(_fp8_problem(name))


def test_fp8_forward_nan_in_unused_kv_rows():
    p = _poison_unused_kv(_fp8_problem("fp8_paged"))
    assert torch.isnan(p.k.float()).any()
    _check_fp8(p)


def test_fp8_pack_is_round_to_nearest_even():
    """The kernel's P packing against torch's fp32 -> e4m3 conversion, byte
    order included; out-of-range values saturate to +-448."""
    g = torch.Generator().manual_seed(5)
    x = torch.cat([torch.randn(4096, generator=g) * 4,
                   torch.rand(4096, generator=g) * 2.0 ** -6,         # subnormal range
                   torch.tensor([0.0, -0.0, 448.0, -448.0, 2.0 ** -10, 3 * 2.0 ** -10,
                                 1.0625, 1.1875, 240.0, 2.0 ** -9])])
    x = x[: (x.numel() // 4) * 4]
    got = bsa.bsa_selftest_e4m3(x.cuda()).cpu()
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8)
    assert torch.equal(got, ref)
    sat = bsa.bsa_selftest_e4m3(torch.tensor([1000.0, -1000.0, 449.0, 0.5]).cuda()).cpu()
    assert sat.tolist() == [0x7E, 0xFE, 0x7E, 0x30]
