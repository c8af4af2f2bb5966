"""Dense, mask-based attention built from torch library routines (fp64).

Used only to pin the oracle: the block index is expanded into a boolean
token mask (the BlockSparseAttentionGrad blockSparseMask form: 1 = the
block takes part), and attention is then torch's own matmul / softmax /
logsumexp / autograd on that mask.  Nothing here shares code with the
oracle's row-by-row C loops.
"""
from __future__ import annotations

import numpy as np
import torch


def _lens(p):
    if p.layout_q == "TND":
        cu = p.cu_q.tolist()
        qs = [(cu[b], cu[b + 1] - cu[b]) for b in range(p.B)]
    else:
        qs = [(0, p.q.shape[2])] * p.B
    if p.seqused_kv is not None:
        kl = [int(x) for x in p.seqused_kv]
    elif p.layout_kv == "TND":
        cu = p.cu_kv.tolist()
        kl = [cu[b + 1] - cu[b] for b in range(p.B)]
    else:
        kl = [p.k.shape[2]] * p.B
    return qs, kl


def batch_tensors(p, b, q, k, v):
    """(q_b [N1, qlen, D], k_b [N2, kvlen, D], v_b) for batch b, any layout."""
    qs, kl = _lens(p)
    s0, L = qs[b]
    kvlen = kl[b]
    qb = q[b] if p.layout_q == "BNSD" else q[s0:s0 + L].transpose(0, 1)
    if p.layout_kv == "BNSD":
        kb, vb = k[b, :, :kvlen], v[b, :, :kvlen]
    elif p.layout_kv == "TND":
        c0 = int(p.cu_kv[b])
        kb, vb = k[c0:c0 + kvlen].transpose(0, 1), v[c0:c0 + kvlen].transpose(0, 1)
    else:
        ps = k.shape[1]
        pages = p.block_table[b, :(kvlen + ps - 1) // ps].long()
        kb = k[pages].reshape(-1, p.N2, p.D)[:kvlen].transpose(0, 1)
        vb = v[pages].reshape(-1, p.N2, p.D)[:kvlen].transpose(0, 1)
    return qb, kb, vb


def token_mask(p, b):
    """[N1, qlen, kvlen] bool: the index rows of batch b expanded to tokens."""
    qs, kl = _lens(p)
    L, kvlen = qs[b][1], kl[b]
    idx = p.index.view(torch.int16).numpy().view(np.uint16)
    g = p.N1 // p.N2
    nq = -(-L // p.BQ)
    qoff = sum(-(-qs[bb][1] // p.BQ) for bb in range(b)) if p.layout_q == "TND" else 0
    m = torch.zeros(p.N1, L, kvlen, dtype=torch.bool)
    for h1 in range(p.N1):
        hi = h1 if p.Hidx == p.N1 else h1 // g
        for i in range(nq):
            row = idx[b, hi, i] if p.layout_q == "BNSD" else idx[hi, qoff + i]
            for e in row:
                if e != 0xFFFF:
                    m[h1, i * p.BQ:(i + 1) * p.BQ, int(e) * p.BKV:(int(e) + 1) * p.BKV] = True
    if getattr(p, "causal", False):
        # the causal mask, aligned to the end of the kv sequence
        t = torch.arange(L).view(L, 1)
        u = torch.arange(kvlen).view(1, kvlen)
        m &= (u <= t + (kvlen - L)).unsqueeze(0)
    return m


def attention(p, q=None, k=None, v=None):
    """Per-batch list of (out [N1, qlen, D], lse [N1, qlen]) in fp64 via torch ops."""
    q = (p.q if q is None else q).double()
    k = (p.k if k is None else k).double()
    v = (p.v if v is None else v).double()
    g = p.N1 // p.N2
    res = []
    for b in range(p.B):
        qb, kb, vb = batch_tensors(p, b, q, k, v)
        kb = kb.repeat_interleave(g, 0)
        vb = vb.repeat_interleave(g, 0)
        s = p.scale * torch.matmul(qb, kb.transpose(-1, -2))
        s = s.masked_fill(~token_mask(p, b), float("-inf"))
        lse = torch.logsumexp(s, -1)
        pr = torch.softmax(s, -1)
        pr = torch.nan_to_num(pr, nan=0.0)     # a row with no selected token
        res.append((torch.matmul(pr, vb), lse))
    return res


def to_q_layout(p, per_batch, which=0):
    """Scatter per-batch results back into the q layout (which=0 out, 1 lse)."""
    if which == 0:
        dst = torch.zeros(p.q.shape, dtype=torch.float64)
    else:
        shape = (p.B, p.N1, p.q.shape[2]) if p.layout_q == "BNSD" else (p.q.shape[0], p.N1)
        dst = torch.full(shape, float("-inf"), dtype=torch.float64)
    qs, _ = _lens(p)
    for b, r in enumerate(per_batch):
        x = r[which]
        if p.layout_q == "BNSD":
            dst[b] = x
        else:
            s0, L = qs[b]
            dst[s0:s0 + L] = x.transpose(0, 1)
    return dst


def grads(p, dout):
    """torch autograd of L = sum(dOut * out) -> (dq, dk, dv) in the input layouts."""
    q = p.q.double().clone().requires_grad_(True)
    k = p.k.double().clone().requires_grad_(True)
    v = p.v.double().clone().requires_grad_(True)
    per = attention(p, q, k, v)
    qs, _ = _lens(p)
    loss = 0.0
    d = dout.double()
    for b, (ob, _) in enumerate(per):
        if p.layout_q == "BNSD":
            loss = loss + (ob * d[b]).sum()
        else:
            s0, L = qs[b]
            loss = loss + (ob * d[s0:s0 + L].transpose(0, 1)).sum()
    loss.backward()
    return q.grad, k.grad, v.grad
