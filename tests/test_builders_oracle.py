"""Pins for the builder oracle (compacted rows, inverted index, work lists):
a case worked by hand, and brute force through the token-mask form on
random tiny problems."""
import json
import os

import numpy as np
import pytest
import torch

from oracle import builders
from workloads.gen import make_problem, pat_density, pat_random_k
from tests import torch_reference as tr

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _hand_problem():
    g = json.load(open(os.path.join(GOLDEN, "builders_hand_case.json")))
    pr = dict(g["problem"])
    p = make_problem(pattern=pat_random_k, **pr)
    idx = np.array(g["index"], dtype=np.uint16)
    p.index = torch.from_numpy(idx.view(np.int16)).view(torch.uint16)
    return p, g["expect"]


def test_hand_worked_case():
    p, e = _hand_problem()
    out = builders.build_all(p)
    geo = out["geo"]
    assert out["flags"] == e["flags"]
    assert geo.qoff == e["qoff"] and geo.koff == e["koff"]
    assert geo.Rg == e["Rg"] and geo.TK == e["TK"]
    assert out["ncomp"].tolist() == e["ncomp"]
    assert out["comp"].tolist() == e["comp"]
    assert out["inv_off"].tolist() == e["inv_off"]
    assert out["inv_list"].tolist() == e["inv_list"]
    assert out["fwd_items"].tolist() == e["fwd_items"]
    assert {str(i): int(out["fwd_cost"][i]) for i in out["fwd_items"]} == e["fwd_cost_of_item"]
    assert out["bwd_items"].tolist() == e["bwd_items"]
    assert {str(i): int(out["bwd_cost"][i]) for i in out["bwd_items"]} == e["bwd_cost_of_item"]
    assert builders.pairs(p, geo, out["comp"], out["ncomp"]) == e["pairs"]


RANDOM = [
    dict(layout_q="TND", layout_kv="TND", B=3, N1=4, N2=2, D=16, BQ=256, BKV=128,
         lens_q=[300, 1, 530], lens_kv=[700, 90, 129], pattern=pat_density(0.4)),
    dict(layout_q="TND", layout_kv="TND", B=2, N1=4, N2=2, Hidx=2, D=16, BQ=128, BKV=256,
         lens_q=[257, 640], lens_kv=[513, 100], pattern=pat_random_k),
    dict(layout_q="BNSD", layout_kv="BNSD", B=2, N1=3, N2=1, D=16, BQ=128, BKV=512, Sq=700,
         lens_kv=[1100, 333], Skv=1200, pattern=pat_density(0.6)),
    dict(layout_q="TND", layout_kv="PA_BBND", B=3, N1=2, N2=2, D=16, BQ=128, BKV=128,
         lens_q=[200, 300, 129], lens_kv=[500, 128, 1], page_size=128, pattern=pat_random_k),
    # the group shares its index row, g = 4 and g = 8: packed forward items
    dict(layout_q="TND", layout_kv="TND", B=3, N1=8, N2=2, Hidx=2, D=16, BQ=256, BKV=128,
         lens_q=[300, 20, 530], lens_kv=[700, 90, 129], pattern=pat_density(0.5)),
    dict(layout_q="BNSD", layout_kv="BNSD", B=2, N1=8, N2=1, Hidx=1, D=16, BQ=128, BKV=256,
         Sq=300, lens_kv=[600, 257], Skv=600, pattern=pat_random_k),
]


def _bwd_order(bcost, N2, per_head, ksl):
    """The backward order from item costs alone: items above 1/512 of the
    total (every kv block counted at full length: slice 0's cost times the
    slices per block) first by cost; then per kv head, by cost within it."""
    total = sum(c * ksl for i, c in bcost.items() if i % ksl == 0)
    big = total >> 9 if N2 <= 1024 else -1

    def key(i):
        c = bcost[i]
        return (0, 0, -c, i) if c > big else (1, i // per_head, -min(c, (1 << 21) - 1), i)
    return sorted(bcost, key=key)


def test_bwd_order_groups_small_items_by_kv_head():
    """With many kv heads the total is large enough that most items fall
    below 1/512 of it: those follow head by head, after the large ones;
    costs counted here from the raw index rows (distinct in-range entries)."""
    from workloads.gen import pat_sink_diag_random
    p = make_problem(B=1, N1=48, N2=48, D=64, Sq=2048, BQ=128, BKV=128, W=8,
                     pattern=pat_sink_diag_random(5), seed_base=321)
    out = builders.build_all(p)
    idx = p.index.view(torch.int16).numpy().view(np.uint16)
    nq = nk = 2048 // 128
    bcost = {}
    for h in range(p.N2):
        for j in range(nk):
            bcost[h * nk + j] = sum(1 for i in range(nq)
                                    if j in {int(e) for e in idx[0, h, i] if int(e) < nk})
    want = _bwd_order(bcost, p.N2, nk, 1)
    assert out["bwd_items"].tolist() == want
    total = sum(bcost.values())
    small = [i for i in want if bcost[i] <= total >> 9]
    assert 0 < len(small) < len(want)            # both parts present
    heads = [i // nk for i in small]
    assert heads == sorted(heads)                # the small items head by head


@pytest.mark.parametrize("case", range(len(RANDOM)))
def test_brute_force_token_mask(case):
    """Compaction == sorted distinct entries; inverse == transpose of the
    token mask; costs == distinct 128-slices touched; order == sorted()."""
    p = make_problem(seed_base=100 + case, **RANDOM[case])
    out = builders.build_all(p)
    geo = out["geo"]
    assert out["flags"] == 0
    g = p.N1 // p.N2
    idx = p.index.view(torch.int16).numpy().view(np.uint16)
    inv = {}
    fcost = {}
    bcost = {}
    nsub, ksl = p.BQ // 128, p.BKV // 128
    for b in range(p.B):
        m = tr.token_mask(p, b).numpy()          # [N1, qlen, kvlen]
        qlen, kvlen = geo.qlen[b], geo.kvlen[b]
        for h1 in range(p.N1):
            hi = h1 if p.Hidx == p.N1 else h1 // g
            for i in range(geo.nq[b]):
                gq = geo.qoff[b] + i
                raw = idx[b, hi, i] if p.layout_q == "BNSD" else idx[hi, gq]
                want = sorted(set(int(x) for x in raw) - {0xFFFF})
                n = out["ncomp"][hi, gq]
                assert out["comp"][hi, gq, :n].tolist() == want
                for qs in range(nsub):
                    t = i * p.BQ + qs * 128
                    if t < qlen:
                        slices = {u // 128 for u in np.nonzero(m[h1, t])[0]}
                        fcost[(h1 * geo.Rg + gq) * nsub + qs] = len(slices)
                for j in want:
                    inv.setdefault((hi, geo.koff[b] + j), set()).add(i)
        for j in range(geo.nk[b]):
            gk = geo.koff[b] + j
            for h2 in range(p.N2):
                c = 0
                for h1 in range(h2 * g, (h2 + 1) * g):
                    rows = np.nonzero(m[h1, :, j * p.BKV])[0]
                    c += len({t // 128 for t in rows})
                for ks in range(ksl):
                    if j * p.BKV + ks * 128 < kvlen:
                        bcost[(h2 * geo.TK + gk) * ksl + ks] = c
    off, lst = out["inv_off"], out["inv_list"]
    for hi in range(p.Hidx):
        for gk in range(geo.TK):
            li = hi * geo.TK + gk
            assert lst[off[li]:off[li + 1]].tolist() == sorted(inv.get((hi, gk), set()))
    want_f = [i for _, i in sorted((-c, i) for i, c in fcost.items())]
    assert out["fwd_items_per_head"].tolist() == want_f
    assert out["bwd_items"].tolist() == _bwd_order(bcost, p.N2, geo.TK * ksl, ksl)
    # packed heads (the group shares its index row): one item per run of
    # 128/g rows of a q block for all g heads, cost from the token mask of
    # the group's first head at the run's first row
    if p.Hidx == p.N2 and g in (2, 4, 8, 16):
        R = 128 // g
        fsub = p.BQ // R
        pcost = {}
        for b in range(p.B):
            m = tr.token_mask(p, b).numpy()
            for h2 in range(p.N2):
                for i in range(geo.nq[b]):
                    gq = geo.qoff[b] + i
                    for s in range(fsub):
                        t = i * p.BQ + s * R
                        if t < geo.qlen[b]:
                            pcost[(h2 * geo.Rg + gq) * fsub + s] = len(
                                {u // 128 for u in np.nonzero(m[h2 * g, t])[0]})
        assert out["fwd_items"].tolist() == [i for _, i in sorted((-c, i) for i, c in pcost.items())]
    else:
        assert out["fwd_items"].tolist() == want_f
