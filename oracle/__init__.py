"""CPU oracle for block-sparse variable-length attention.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` / ``--impl reference`` legs are the only
callers.  The product library never imports this package and this package
never imports the product.  Inputs come from ``workloads`` (random draws
only); all arithmetic here is the plain definition in fp64
(``bsa_oracle.c``) plus the index/work-list builders in ``builders.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bsa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

LAYOUT = {"BNSD": 0, "TND": 1, "PA_BBND": 2}
BAD_INDEX, BAD_SEQLEN, BAD_PAGE = 1, 2, 4


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c99",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Problem(ctypes.Structure):
    _fields_ = [("layout_q", ctypes.c_int32), ("layout_kv", ctypes.c_int32),
                ("B", ctypes.c_int64), ("N1", ctypes.c_int64), ("N2", ctypes.c_int64),
                ("D", ctypes.c_int64), ("Sq", ctypes.c_int64), ("Skv", ctypes.c_int64),
                ("Tq", ctypes.c_int64), ("Tkv", ctypes.c_int64),
                ("num_pages", ctypes.c_int64), ("page_size", ctypes.c_int64),
                ("max_pages", ctypes.c_int64),
                ("BQ", ctypes.c_int64), ("BKV", ctypes.c_int64), ("Hidx", ctypes.c_int64),
                ("R", ctypes.c_int64), ("W", ctypes.c_int64), ("scale", ctypes.c_double),
                ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("index", ctypes.c_void_p), ("cu_q", ctypes.c_void_p), ("cu_kv", ctypes.c_void_p),
                ("seqused_kv", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
                ("causal", ctypes.c_int32)]


_lib = None


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.POINTER(_Problem)
        vp, i64 = ctypes.c_void_p, ctypes.c_int64
        _lib.oracle_fwd_rows.argtypes = [P, vp, i64, vp, vp, vp]
        _lib.oracle_bwd_dq_rows.argtypes = [P, vp, vp, vp, vp, i64, vp, vp]
        _lib.oracle_bwd_dkv_rows.argtypes = [P, vp, vp, vp, vp, i64, vp, vp, vp]
        _lib.oracle_scan_flags.argtypes = [P, vp]
        _lib.oracle_batch_lengths.argtypes = [P, vp, vp, vp, vp]
    return _lib


def _f64(t: torch.Tensor) -> np.ndarray:
    return np.ascontiguousarray(t.detach().to(torch.float64).cpu().numpy())


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


class Oracle:
    """Binds one ``workloads.Problem`` (inputs converted exactly to fp64)."""

    def __init__(self, prob, q=None, k=None, v=None):
        self.prob = prob
        p = prob
        self._keep = {
            "q": _f64(p.q if q is None else q), "k": _f64(p.k if k is None else k),
            "v": _f64(p.v if v is None else v),
            "index": np.ascontiguousarray(p.index.view(torch.int16).numpy()).view(np.uint16),
            "cu_q": None if p.cu_q is None else np.ascontiguousarray(p.cu_q.numpy().astype(np.int64)),
            "cu_kv": None if p.cu_kv is None else np.ascontiguousarray(p.cu_kv.numpy().astype(np.int64)),
            "seqused_kv": None if p.seqused_kv is None else np.ascontiguousarray(p.seqused_kv.numpy().astype(np.int32)),
            "block_table": None if p.block_table is None else np.ascontiguousarray(p.block_table.numpy().astype(np.int32)),
        }
        K = self._keep
        s = _Problem()
        s.layout_q, s.layout_kv = LAYOUT[p.layout_q], LAYOUT[p.layout_kv]
        s.B, s.N1, s.N2, s.D = p.B, p.N1, p.N2, p.D
        s.Sq = p.q.shape[2] if p.layout_q == "BNSD" else 0
        s.Tq = p.q.shape[0] if p.layout_q == "TND" else 0
        s.Skv = p.k.shape[2] if p.layout_kv == "BNSD" else 0
        s.Tkv = p.k.shape[0] if p.layout_kv == "TND" else 0
        if p.layout_kv == "PA_BBND":
            s.num_pages, s.page_size, s.max_pages = p.k.shape[0], p.k.shape[1], p.block_table.shape[1]
        s.BQ, s.BKV, s.Hidx = p.BQ, p.BKV, p.Hidx
        s.R, s.W = p.index.shape[-2], p.index.shape[-1]
        s.scale = p.scale
        s.q, s.k, s.v, s.index = (K[n].ctypes.data for n in ("q", "k", "v", "index"))
        s.cu_q, s.cu_kv = _ptr(K["cu_q"]), _ptr(K["cu_kv"])
        s.seqused_kv, s.block_table = _ptr(K["seqused_kv"]), _ptr(K["block_table"])
        s.causal = int(bool(getattr(p, "causal", False)))
        self._s = s
        self.lib = _load()

    # ---------------------------------------------------------- lengths
    def batch_lengths(self):
        """Per batch (query rows, used kv tokens, stored kv rows) and the flag
        bits the lengths raise; a length that contradicts its storage counts
        as 0 (bsa_oracle.c, oracle_batch_lengths)."""
        B = self.prob.B
        ql, kl, ks = (np.zeros(B, np.int64) for _ in range(3))
        fl = ctypes.c_uint32(0)
        self.lib.oracle_batch_lengths(ctypes.byref(self._s), ql.ctypes.data, kl.ctypes.data,
                                      ks.ctypes.data, ctypes.addressof(fl))
        return [int(x) for x in ql], [int(x) for x in kl], [int(x) for x in ks], fl.value

    # ------------------------------------------------------------- rows
    def q_rows_all(self) -> np.ndarray:
        """All (b, h1, t) query rows of every batch (t below the batch's query
        length), in storage order of the q tensor's rows."""
        p = self.prob
        rows = []
        if p.layout_q == "BNSD":
            S = p.q.shape[2]
            b, h, t = np.meshgrid(np.arange(p.B), np.arange(p.N1), np.arange(S), indexing="ij")
            return np.stack([b.ravel(), h.ravel(), t.ravel()], 1).astype(np.int64)
        qlen = self.batch_lengths()[0]
        for b in range(p.B):
            L = qlen[b]
            t, h = np.meshgrid(np.arange(L), np.arange(p.N1), indexing="ij")
            rows.append(np.stack([np.full(t.size, b), h.ravel(), t.ravel()], 1))
        return np.concatenate(rows).astype(np.int64) if rows else np.zeros((0, 3), np.int64)

    def fwd_rows(self, rows: np.ndarray) -> Tuple[np.ndarray, np.ndarray, int]:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        n = rows.shape[0]
        out = np.zeros((n, self.prob.D))
        lse = np.zeros(n)
        fl = ctypes.c_uint32(0)
        self.lib.oracle_fwd_rows(ctypes.byref(self._s), rows.ctypes.data, n, out.ctypes.data,
                                 lse.ctypes.data, ctypes.addressof(fl))
        return out, lse, fl.value

    def fwd(self) -> Tuple[torch.Tensor, torch.Tensor, int]:
        """Full forward: out (q layout, fp64) and lse ([B,N1,Sq] or [Tq,N1], fp64)."""
        p = self.prob
        rows = self.q_rows_all()
        o, l, fl = self.fwd_rows(rows)
        out = torch.zeros(p.q.shape, dtype=torch.float64)
        lse = torch.full(self.lse_shape(), float("-inf"), dtype=torch.float64)
        self._scatter_q(out, rows, torch.from_numpy(o))
        self._scatter_stat(lse, rows, torch.from_numpy(l))
        return out, lse, fl

    def lse_shape(self):
        p = self.prob
        return (p.B, p.N1, p.q.shape[2]) if p.layout_q == "BNSD" else (p.q.shape[0], p.N1)

    def _scatter_q(self, dst, rows, vals):
        p = self.prob
        b, h, t = (torch.from_numpy(rows[:, i]) for i in range(3))
        if p.layout_q == "BNSD":
            dst[b, h, t] = vals
        else:
            dst[p.cu_q[b] + t, h] = vals

    def _scatter_stat(self, dst, rows, vals):
        p = self.prob
        b, h, t = (torch.from_numpy(rows[:, i]) for i in range(3))
        if p.layout_q == "BNSD":
            dst[b, h, t] = vals
        else:
            dst[p.cu_q[b] + t, h] = vals

    def gather_q(self, src: torch.Tensor, rows: np.ndarray) -> torch.Tensor:
        """Rows of a q-layout tensor (or lse-layout tensor) at (b, h1, t)."""
        p = self.prob
        b, h, t = (torch.from_numpy(np.ascontiguousarray(rows[:, i])) for i in range(3))
        if p.layout_q == "BNSD":
            return src[b, h, t]
        return src[p.cu_q[b] + t, h]

    # --------------------------------------------------------- backward
    def _bwd_inputs(self, out, dout, lse):
        return _f64(out), _f64(dout), _f64(lse)

    def bwd_dq_rows(self, out, dout, lse, rows):
        o, d, l = self._bwd_inputs(out, dout, lse)
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        dq = np.zeros((rows.shape[0], self.prob.D))
        fl = ctypes.c_uint32(0)
        self.lib.oracle_bwd_dq_rows(ctypes.byref(self._s), o.ctypes.data, d.ctypes.data,
                                    l.ctypes.data, rows.ctypes.data, rows.shape[0],
                                    dq.ctypes.data, ctypes.addressof(fl))
        return dq, fl.value

    def bwd_dkv_rows(self, out, dout, lse, kvrows):
        o, d, l = self._bwd_inputs(out, dout, lse)
        kvrows = np.ascontiguousarray(kvrows, dtype=np.int64)
        n = kvrows.shape[0]
        dk = np.zeros((n, self.prob.D))
        dv = np.zeros((n, self.prob.D))
        fl = ctypes.c_uint32(0)
        self.lib.oracle_bwd_dkv_rows(ctypes.byref(self._s), o.ctypes.data, d.ctypes.data,
                                     l.ctypes.data, kvrows.ctypes.data, n, dk.ctypes.data,
                                     dv.ctypes.data, ctypes.addressof(fl))
        return dk, dv, fl.value

    def kv_rows_all(self) -> np.ndarray:
        """All (b, h2, u) kv rows with u < the batch's used kv length (paged:
        whose block-table entry names a page; the tokens of a bad entry have
        no storage row)."""
        p = self.prob
        lens = self.kv_lens()
        rows = []
        for b in range(p.B):
            us = np.arange(lens[b])
            if p.layout_kv == "PA_BBND":
                pages = p.block_table[b].numpy().astype(np.int64)[us // p.k.shape[1]]
                us = us[(pages >= 0) & (pages < p.k.shape[0])]
            u, h = np.meshgrid(us, np.arange(p.N2), indexing="ij")
            rows.append(np.stack([np.full(u.size, b), h.ravel(), u.ravel()], 1))
        return np.concatenate(rows).astype(np.int64) if rows else np.zeros((0, 3), np.int64)

    def kv_lens(self):
        """Used kv tokens per batch (0 where a length contradicts its storage)."""
        return self.batch_lengths()[1]

    def kv_index(self, kvrows: np.ndarray):
        """Advanced-index tuple addressing kv rows (b, h2, u) in the k/v tensor."""
        p = self.prob
        b, h, u = (torch.from_numpy(np.ascontiguousarray(kvrows[:, i])) for i in range(3))
        if p.layout_kv == "BNSD":
            return (b, h, u)
        if p.layout_kv == "TND":
            return (p.cu_kv[b] + u, h)
        pg = p.block_table[b, u // p.page_size].long()
        return (pg, u % p.page_size, h)

    def bwd(self, out, dout, lse):
        """Full backward: dq (q layout), dk / dv (kv layout; untouched kv rows 0)."""
        p = self.prob
        rows = self.q_rows_all()
        dq_r, f1 = self.bwd_dq_rows(out, dout, lse, rows)
        kvr = self.kv_rows_all()
        dk_r, dv_r, f2 = self.bwd_dkv_rows(out, dout, lse, kvr)
        dq = torch.zeros(p.q.shape, dtype=torch.float64)
        self._scatter_q(dq, rows, torch.from_numpy(dq_r))
        dk = torch.zeros(p.k.shape, dtype=torch.float64)
        dv = torch.zeros(p.v.shape, dtype=torch.float64)
        ix = self.kv_index(kvr)
        dk[ix] = torch.from_numpy(dk_r)
        dv[ix] = torch.from_numpy(dv_r)
        return dq, dk, dv, f1 | f2

    def scan_flags(self) -> int:
        fl = ctypes.c_uint32(0)
        self.lib.oracle_scan_flags(ctypes.byref(self._s), ctypes.addressof(fl))
        return fl.value
