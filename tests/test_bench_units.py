"""The benchmark's algorithmic unit: kept (q head, valid q token, visible kv
token) pairs.  bench._pairs counts them from the index arithmetically; here
the count is checked against the dense token mask (torch_reference) on small
problems of every layout, with and without the causal mask, and the causal
C3 closed form S(S+1)/2 per head."""
import sys
import os

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from tests import torch_reference as TR  # noqa: E402
from workloads.gen import (make_problem, pat_causal, pat_causal_blocks, pat_dense,  # noqa: E402
                           pat_fraction_diag, pat_random_k, pat_topk)

CASES = {
    "bnsd": dict(layout_q="BNSD", layout_kv="BNSD", B=2, N1=2, N2=1, D=16, Sq=300,
                 lens_kv=[300, 170], Skv=300, pattern=pat_random_k),
    "bnsd_blocks": dict(layout_q="BNSD", layout_kv="BNSD", B=1, N1=2, N2=2, D=16, Sq=700, BQ=256,
                        BKV=512, pattern=pat_dense),
    "tnd_gqa_shared": dict(layout_q="TND", layout_kv="TND", B=3, N1=4, N2=2, Hidx=2, D=16,
                           lens_q=[130, 300, 77], lens_kv=[200, 129, 256],
                           pattern=pat_fraction_diag(0.5)),
    "paged": dict(layout_q="TND", layout_kv="PA_BBND", B=2, N1=2, N2=1, D=16,
                  lens_q=[300, 129], lens_kv=[456, 129], page_size=128, pattern=pat_topk(2)),
}


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("name", sorted(CASES))
def test_pairs_count_the_dense_mask(name, causal):
    p = make_problem(seed_base=11, causal=causal, **CASES[name])
    dense = sum(int(TR.token_mask(p, b).sum()) for b in range(p.B))
    assert bench._pairs(p) == dense


def test_causal_square_closed_form():
    S = 1024
    p = make_problem(layout_q="BNSD", layout_kv="BNSD", B=1, N1=3, N2=3, D=16, Sq=S, BQ=128, BKV=512,
                     pattern=pat_causal_blocks(128, 512), causal=True, seed_base=3)
    assert bench._pairs(p) == 3 * S * (S + 1) // 2
    q = make_problem(layout_q="BNSD", layout_kv="BNSD", B=1, N1=1, N2=1, D=16, Sq=S, BQ=128, BKV=128,
                     pattern=pat_causal, causal=True, seed_base=3)
    assert bench._pairs(q) == S * (S + 1) // 2


def test_causal_blocks_pattern_is_exactly_the_reachable_blocks():
    """C3's causal variant keeps, for query block i, exactly the kv blocks
    that hold at least one token a row of block i may see."""
    S, BQ, BKV = 2048, 128, 512
    p = make_problem(layout_q="BNSD", layout_kv="BNSD", B=1, N1=1, N2=1, D=16, Sq=S, BQ=BQ, BKV=BKV,
                     pattern=pat_causal_blocks(BQ, BKV), causal=True, seed_base=5)
    idx = p.index.view(torch.int16).numpy().view("uint16")[0, 0]
    for i in range(S // BQ):
        row = sorted(int(e) for e in idx[i] if e != 0xFFFF)
        last_visible = i * BQ + BQ - 1          # the block's last row sees up to its own token
        want = list(range(last_visible // BKV + 1))
        assert row == want, (i, row, want)


def test_oracle_sample_takes_whole_heads_past_one_head():
    """The CPU-baseline slice of C3 (dense index, S = 8192) grows by whole
    heads once it asks for more rows than one head holds: each head keeps all
    S x S pairs, and its tensors are the workload's own heads 0..h-1."""
    sub = bench._oracle_subproblem(3, 3 * 8192 + 100)
    assert sub.N1 == sub.N2 == 3 and sub.q.shape[1:3] == (3, 8192)
    assert bench._pairs(sub) == 3 * 8192 * 8192
    one = bench._oracle_subproblem(3, 1024)
    assert one.N1 == 1 and bench._pairs(one) == 1024 * 8192
    assert torch.equal(one.q[0, 0], sub.q[0, 0, :1024])


def test_launch_count_follows_the_sort_chunks():
    """One sort launch for a list of up to 4096 slots, a sort and a rank
    merge above; C3's lists have 4096 slots each, C4's 6144."""
    assert bench.launches_per_step(4096, 4096, False) == 15
    assert bench.launches_per_step(6144, 6144, False) == 17
    assert bench.launches_per_step(4096, 4096, True) == 16
    assert bench.launches_per_step(6144, 6144, True) == 19
