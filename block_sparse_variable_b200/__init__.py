"""Block-sparse variable-length FlashAttention for B200 (sm_100a).

Thin ctypes binding over the C ABI in ``include/bsa.h`` (``libbsa.so``,
built in-tree by ``block_sparse_variable_b200/build.py``).  The functions keep
the C names; they only marshal torch tensors into ``bsa_tensor``
descriptors, allocate outputs / workspace with torch when the caller does
not pass them, and raise ``BsaError`` on a non-OK status.  Every step of
the computation runs in the library's CUDA kernels: there is no fallback,
and importing this package fails if the library is missing.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbsa.so")

BSA_F16, BSA_BF16, BSA_F32, BSA_U16, BSA_I32, BSA_I64, BSA_F8E4M3 = 1, 2, 3, 4, 5, 6, 7
LAYOUTS = {"BNSD": 0, "TND": 1, "PA_BBND": 2}
FLAG_BAD_INDEX, FLAG_BAD_SEQLEN, FLAG_BAD_PAGE, FLAG_TIMEOUT = 1, 2, 4, 8
STATUS_NAMES = {0: "BSA_OK", 161001: "BSA_ERR_NULLPTR", 161002: "BSA_ERR_PARAM_INVALID",
                161003: "BSA_ERR_UNSUPPORTED", 161004: "BSA_ERR_WORKSPACE",
                561000: "BSA_ERR_CUDA", 561103: "BSA_ERR_INNER"}

_DTYPES = {torch.float16: BSA_F16, torch.bfloat16: BSA_BF16, torch.float32: BSA_F32,
           torch.uint16: BSA_U16, torch.int32: BSA_I32, torch.int64: BSA_I64,
           torch.float8_e4m3fn: BSA_F8E4M3}


class BsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


class bsa_tensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class bsa_params(ctypes.Structure):
    _fields_ = [("q_layout", ctypes.c_int32), ("kv_layout", ctypes.c_int32),
                ("num_heads", ctypes.c_int64), ("num_kv_heads", ctypes.c_int64),
                ("block_shape", ctypes.c_int64 * 2), ("scale", ctypes.c_double),
                ("return_lse", ctypes.c_int32), ("mask_type", ctypes.c_int32),
                ("deterministic", ctypes.c_int32)]


class bsa_ws_region(ctypes.Structure):
    _fields_ = [("offset", ctypes.c_uint64), ("bytes", ctypes.c_uint64)]


class bsa_ws_layout(ctypes.Structure):
    _fields_ = [(n, bsa_ws_region) for n in ("status", "batch", "comp", "ncomp", "fwd_items",
                                              "inv_off", "inv_list", "bwd_items", "dsum",
                                              "dq_acc", "sort_keys")] + \
               [("Rg", ctypes.c_int64), ("tk_max", ctypes.c_int64), ("total_bytes", ctypes.c_uint64)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          f"`python block_sparse_variable_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    T = ctypes.POINTER(bsa_tensor)
    Pp = ctypes.POINTER(bsa_params)
    L = ctypes.POINTER(bsa_ws_layout)
    sz = ctypes.POINTER(ctypes.c_size_t)
    vp, s_t = ctypes.c_void_p, ctypes.c_size_t
    lib.bsa_fwd_get_workspace.argtypes = [T] * 8 + [Pp, T, T, sz]
    lib.bsa_fwd.argtypes = [T] * 8 + [Pp, T, T, vp, s_t, vp]
    lib.bsa_fwd_workspace_layout.argtypes = [T] * 8 + [Pp, T, T, L]
    lib.bsa_bwd_get_workspace.argtypes = [T] * 11 + [Pp, T, T, T, sz]
    lib.bsa_bwd.argtypes = [T] * 11 + [Pp, T, T, T, vp, s_t, vp]
    lib.bsa_bwd_workspace_layout.argtypes = [T] * 11 + [Pp, T, T, T, L]
    lib.bsa_read_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.bsa_status_string.argtypes = [ctypes.c_int]
    lib.bsa_status_string.restype = ctypes.c_char_p
    lib.bsa_abi_version.restype = ctypes.c_int32
    lib.bsa_set_main_kernel_events.argtypes = [vp, vp]
    lib.bsa_selftest_exp2.argtypes = [vp, vp, vp, ctypes.c_int64, vp]
    lib.bsa_selftest_e4m3.argtypes = [vp, vp, ctypes.c_int64, vp]
    lib.bsa_selftest_wait_timeout.argtypes = [vp, vp]
    lib.bsa_selftest_f32x2.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int64, vp]
    for f in ("bsa_fwd_get_workspace", "bsa_fwd", "bsa_fwd_workspace_layout",
              "bsa_bwd_get_workspace", "bsa_bwd", "bsa_bwd_workspace_layout", "bsa_read_status",
              "bsa_set_main_kernel_events", "bsa_selftest_exp2", "bsa_selftest_wait_timeout",
              "bsa_selftest_e4m3", "bsa_selftest_f32x2"):
        getattr(lib, f).restype = ctypes.c_int
    return lib


_lib = _load()

EXPORTED = ("bsa_fwd_get_workspace", "bsa_fwd", "bsa_bwd_get_workspace", "bsa_bwd",
            "bsa_read_status", "bsa_status_string", "bsa_fwd_workspace_layout",
            "bsa_bwd_workspace_layout", "bsa_abi_version", "bsa_fwd_static_workspace",
            "bsa_set_main_kernel_events", "bsa_selftest_exp2", "bsa_selftest_wait_timeout",
            "bsa_selftest_e4m3", "bsa_selftest_f32x2")


def lib():
    return _lib


@dataclass
class Params:
    q_layout: str = "BNSD"
    kv_layout: str = "BNSD"
    num_heads: int = 0
    num_kv_heads: int = 0
    block_shape: Tuple[int, int] = (128, 128)
    scale: float = 0.0
    return_lse: bool = True
    causal: bool = False
    deterministic: bool = False

    def c(self) -> bsa_params:
        p = bsa_params()
        p.q_layout, p.kv_layout = LAYOUTS[self.q_layout], LAYOUTS[self.kv_layout]
        p.num_heads, p.num_kv_heads = self.num_heads, self.num_kv_heads
        p.block_shape[0], p.block_shape[1] = self.block_shape
        p.scale = float(self.scale)
        p.return_lse = 1 if self.return_lse else 0
        p.mask_type = 1 if self.causal else 0
        p.deterministic = 1 if self.deterministic else 0
        return p


_EMPTY_PTR = 256  # stand-in address for zero-element and shape-only descriptors


def describe_shape(shape: Sequence[int], dtype: torch.dtype) -> bsa_tensor:
    """A contiguous descriptor with no memory behind it (workspace queries only)."""
    d = bsa_tensor()
    d.data = _EMPTY_PTR
    d.dtype = _DTYPES[dtype]
    d.ndim = len(shape)
    st = 1
    for i in reversed(range(len(shape))):
        d.shape[i] = shape[i]
        d.stride[i] = st
        st *= max(1, shape[i])
    return d


def describe(t: Optional[torch.Tensor]) -> Optional[bsa_tensor]:
    """A bsa_tensor view of a torch tensor (None -> absent)."""
    if t is None:
        return None
    if t.dim() > 4:
        raise ValueError("at most 4 dimensions")
    d = bsa_tensor()
    # an empty tensor may have no storage; nothing is read through it
    d.data = t.data_ptr() or (_EMPTY_PTR if t.numel() == 0 else None)
    d.dtype = _DTYPES.get(t.dtype, 0)
    d.ndim = t.dim()
    for i in range(t.dim()):
        d.shape[i] = t.shape[i]
        d.stride[i] = t.stride(i)
    return d


def _ref(d):
    return None if d is None else ctypes.byref(d)


def _check(st: int, where: str):
    if st != 0:
        raise BsaError(st, where)


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def params_for(q_layout, kv_layout, num_heads, num_kv_heads=0, block_shape=(128, 128), scale=0.0,
               return_lse=True, causal=False, deterministic=False) -> Params:
    return Params(q_layout, kv_layout, int(num_heads), int(num_kv_heads),
                  (int(block_shape[0]), int(block_shape[1])), float(scale), bool(return_lse),
                  bool(causal), bool(deterministic))


def params_of_problem(prob, return_lse=True) -> Params:
    """Params for a problem description: any object with the attributes
    layout_q, layout_kv, N1, N2, BQ, BKV, scale and, optionally, causal and
    deterministic (for example a ``workloads.Problem``)."""
    return params_for(prob.layout_q, prob.layout_kv, prob.N1, prob.N2, (prob.BQ, prob.BKV),
                      prob.scale, return_lse, getattr(prob, "causal", False),
                      getattr(prob, "deterministic", False))


def _fwd_descs(q, k, v, index, cu_seqlens_q, cu_seqlens_kv, seqused_kv, block_table, out, lse):
    return [describe(x) for x in (q, k, v, index, cu_seqlens_q, cu_seqlens_kv, seqused_kv,
                                  block_table)], describe(out), describe(lse)


def _lse_shape(q, params: Params):
    if params.q_layout == "BNSD":
        return (q.shape[0], q.shape[1], q.shape[2])
    return (q.shape[0], q.shape[1])


# ------------------------------------------------------------------ forward
def bsa_fwd_get_workspace(q, k, v, index, params: Params, *, cu_seqlens_q=None, cu_seqlens_kv=None,
                          seqused_kv=None, block_table=None, out=None, lse=None) -> int:
    out = q if out is None else out
    ins, o, l = _fwd_descs(q, k, v, index, cu_seqlens_q, cu_seqlens_kv, seqused_kv, block_table,
                           out, lse)
    if l is None and params.return_lse:
        l = describe_shape(_lse_shape(q, params), torch.float32)
    n = ctypes.c_size_t(0)
    cp = params.c()
    _check(_lib.bsa_fwd_get_workspace(*[_ref(x) for x in ins], ctypes.byref(cp), _ref(o), _ref(l),
                                      ctypes.byref(n)), "bsa_fwd_get_workspace")
    return n.value


def bsa_fwd_workspace_layout(q, k, v, index, params: Params, *, cu_seqlens_q=None,
                             cu_seqlens_kv=None, seqused_kv=None, block_table=None, out=None,
                             lse=None) -> bsa_ws_layout:
    ins, o, l = _fwd_descs(q, k, v, index, cu_seqlens_q, cu_seqlens_kv, seqused_kv, block_table,
                           q if out is None else out, lse)
    lay = bsa_ws_layout()
    cp = params.c()
    _check(_lib.bsa_fwd_workspace_layout(*[_ref(x) for x in ins], ctypes.byref(cp), _ref(o),
                                         _ref(l), ctypes.byref(lay)), "bsa_fwd_workspace_layout")
    return lay


def bsa_fwd(q, k, v, index, params: Params, *, cu_seqlens_q=None, cu_seqlens_kv=None,
            seqused_kv=None, block_table=None, out=None, lse=None, workspace=None, stream=None):
    """Forward pass on the current (or given) stream.  Returns (out, lse, workspace)."""
    if out is None:  # e4m3 inputs: bf16 out unless the caller passes its own
        out = torch.empty_like(q, dtype=torch.bfloat16 if q.dtype == torch.float8_e4m3fn else q.dtype)
    if lse is None and params.return_lse:
        lse = torch.empty(_lse_shape(q, params), dtype=torch.float32, device=q.device)
    ins, o, l = _fwd_descs(q, k, v, index, cu_seqlens_q, cu_seqlens_kv, seqused_kv, block_table,
                           out, lse)
    cp = params.c()
    n = ctypes.c_size_t(0)
    _check(_lib.bsa_fwd_get_workspace(*[_ref(x) for x in ins], ctypes.byref(cp), _ref(o), _ref(l),
                                      ctypes.byref(n)), "bsa_fwd_get_workspace")
    if workspace is None:
        workspace = torch.empty(max(n.value, 256), dtype=torch.uint8, device=q.device)
    _check(_lib.bsa_fwd(*[_ref(x) for x in ins], ctypes.byref(cp), _ref(o), _ref(l),
                        ctypes.c_void_p(workspace.data_ptr()), ctypes.c_size_t(workspace.numel()),
                        ctypes.c_void_p(_stream(stream))), "bsa_fwd")
    return out, lse, workspace


# ----------------------------------------------------------------- backward
def _bwd_descs(q, k, v, out, dout, lse, index, cu_seqlens_q, cu_seqlens_kv, seqused_kv,
               block_table, dq, dk, dv):
    return [describe(x) for x in (q, k, v, out, dout, lse, index, cu_seqlens_q, cu_seqlens_kv,
                                  seqused_kv, block_table)], [describe(x) for x in (dq, dk, dv)]


def bsa_bwd_get_workspace(q, k, v, out, dout, lse, index, params: Params, *, cu_seqlens_q=None,
                          cu_seqlens_kv=None, seqused_kv=None, block_table=None, dq=None, dk=None,
                          dv=None) -> int:
    ins, outs = _bwd_descs(q, k, v, out, dout, lse, index, cu_seqlens_q, cu_seqlens_kv, seqused_kv,
                           block_table, q if dq is None else dq, k if dk is None else dk,
                           v if dv is None else dv)
    n = ctypes.c_size_t(0)
    cp = params.c()
    _check(_lib.bsa_bwd_get_workspace(*[_ref(x) for x in ins], ctypes.byref(cp),
                                      *[_ref(x) for x in outs], ctypes.byref(n)),
           "bsa_bwd_get_workspace")
    return n.value


def bsa_bwd_workspace_layout(q, k, v, out, dout, lse, index, params: Params, *, cu_seqlens_q=None,
                             cu_seqlens_kv=None, seqused_kv=None, block_table=None) -> bsa_ws_layout:
    ins, outs = _bwd_descs(q, k, v, out, dout, lse, index, cu_seqlens_q, cu_seqlens_kv, seqused_kv,
                           block_table, q, k, v)
    lay = bsa_ws_layout()
    cp = params.c()
    _check(_lib.bsa_bwd_workspace_layout(*[_ref(x) for x in ins], ctypes.byref(cp),
                                         *[_ref(x) for x in outs], ctypes.byref(lay)),
           "bsa_bwd_workspace_layout")
    return lay


def bsa_bwd(q, k, v, out, dout, lse, index, params: Params, *, cu_seqlens_q=None,
            cu_seqlens_kv=None, seqused_kv=None, block_table=None, dq=None, dk=None, dv=None,
            workspace=None, stream=None):
    """Backward pass.  Returns (dq, dk, dv, workspace)."""
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    ins, outs = _bwd_descs(q, k, v, out, dout, lse, index, cu_seqlens_q, cu_seqlens_kv, seqused_kv,
                           block_table, dq, dk, dv)
    cp = params.c()
    n = ctypes.c_size_t(0)
    _check(_lib.bsa_bwd_get_workspace(*[_ref(x) for x in ins], ctypes.byref(cp),
                                      *[_ref(x) for x in outs], ctypes.byref(n)),
           "bsa_bwd_get_workspace")
    if workspace is None:
        workspace = torch.empty(max(n.value, 256), dtype=torch.uint8, device=q.device)
    _check(_lib.bsa_bwd(*[_ref(x) for x in ins], ctypes.byref(cp), *[_ref(x) for x in outs],
                        ctypes.c_void_p(workspace.data_ptr()), ctypes.c_size_t(workspace.numel()),
                        ctypes.c_void_p(_stream(stream))), "bsa_bwd")
    return dq, dk, dv, workspace


def bsa_read_status(workspace: torch.Tensor, stream=None) -> int:
    flags = ctypes.c_uint32(0)
    _check(_lib.bsa_read_status(ctypes.c_void_p(workspace.data_ptr()),
                                ctypes.c_void_p(_stream(stream)), ctypes.byref(flags)),
           "bsa_read_status")
    return flags.value


def bsa_status_string(status: int) -> str:
    return _lib.bsa_status_string(int(status)).decode()


def bsa_selftest_exp2(x: torch.Tensor, stream=None):
    """(FMA-pipe 2^x of the softmax kernels, hardware ex2.approx) of a CUDA
    float32 tensor, elementwise."""
    x = x.contiguous()
    yp, ym = torch.empty_like(x), torch.empty_like(x)
    _check(_lib.bsa_selftest_exp2(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(yp.data_ptr()),
                                  ctypes.c_void_p(ym.data_ptr()), x.numel(),
                                  ctypes.c_void_p(_stream(stream))), "bsa_selftest_exp2")
    return yp, ym


def bsa_selftest_e4m3(x: torch.Tensor, stream=None) -> torch.Tensor:
    """Pack a CUDA float32 tensor (numel % 4 == 0) into e4m3 bytes with the
    FP8 forward's routine; returns a uint8 tensor of the same numel."""
    x = x.contiguous()
    y = torch.empty(x.numel() // 4, dtype=torch.int32, device=x.device)
    _check(_lib.bsa_selftest_e4m3(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(y.data_ptr()),
                                  x.numel(), ctypes.c_void_p(_stream(stream))), "bsa_selftest_e4m3")
    return y.view(torch.uint8)


def bsa_selftest_f32x2(a: torch.Tensor, b: torch.Tensor, c: torch.Tensor, stream=None):
    """(paired, scalar) results of fma(a,b,c), a+b and a*b for CUDA float32
    tensors of one even numel; each a float32 tensor [3, numel]."""
    a, b, c = (t.contiguous() for t in (a, b, c))
    n = a.numel()
    pair = torch.empty(3, n, dtype=torch.float32, device=a.device)
    scal = torch.empty_like(pair)
    _check(_lib.bsa_selftest_f32x2(ctypes.c_void_p(a.data_ptr()), ctypes.c_void_p(b.data_ptr()),
                                   ctypes.c_void_p(c.data_ptr()), ctypes.c_void_p(pair.data_ptr()),
                                   ctypes.c_void_p(scal.data_ptr()), n,
                                   ctypes.c_void_p(_stream(stream))), "bsa_selftest_f32x2")
    return pair, scal


def bsa_selftest_wait_timeout(flags: torch.Tensor, stream=None):
    """Run the bounded-wait self test; `flags` is a zeroed int32 CUDA tensor
    whose word 0 receives BSA_FLAG_TIMEOUT."""
    _check(_lib.bsa_selftest_wait_timeout(ctypes.c_void_p(flags.data_ptr()),
                                          ctypes.c_void_p(_stream(stream))),
           "bsa_selftest_wait_timeout")


def bsa_set_main_kernel_events(before=None, after=None):
    """The next bsa_fwd / bsa_bwd of this thread records the two
    torch.cuda.Event objects around its main attention kernel (None, None
    clears).  The events must already exist on the device: record each once
    (on any stream) before handing it over."""
    h = [None if e is None else ctypes.c_void_p(int(e.cuda_event)) for e in (before, after)]
    _check(_lib.bsa_set_main_kernel_events(*h), "bsa_set_main_kernel_events")


# ------------------------------------------------- forward without workspace
STATIC_WORKSPACE_BYTES = 32 << 20


def bsa_fwd_static_workspace(q, k, v, index, params: Params, *, cu_seqlens_q=None,
                             cu_seqlens_kv=None, seqused_kv=None, block_table=None, out=None,
                             lse=None, stream=None):
    """Forward for callers that cannot allocate device memory at run time.

    The library's built-in 32 MiB scratch array replaces the workspace, so
    the call allocates nothing (``out`` / ``lse`` must then be passed in by
    such a caller; they are only created here for convenience when None).
    Calls that may overlap on the GPU share the array and must be
    serialised by the caller.  Returns (out, lse).
    """
    f = _lib.bsa_fwd_static_workspace
    if f.argtypes is None:
        T = ctypes.POINTER(bsa_tensor)
        f.argtypes = [T] * 8 + [ctypes.POINTER(bsa_params), T, T, ctypes.c_void_p]
        f.restype = ctypes.c_int
    if out is None:  # e4m3 inputs: bf16 out unless the caller passes its own
        out = torch.empty_like(q, dtype=torch.bfloat16 if q.dtype == torch.float8_e4m3fn else q.dtype)
    if lse is None and params.return_lse:
        lse = torch.empty(_lse_shape(q, params), dtype=torch.float32, device=q.device)
    ins, o, l = _fwd_descs(q, k, v, index, cu_seqlens_q, cu_seqlens_kv, seqused_kv, block_table,
                           out, lse)
    cp = params.c()
    _check(f(*[_ref(x) for x in ins], ctypes.byref(cp), _ref(o), _ref(l),
             ctypes.c_void_p(_stream(stream))), "bsa_fwd_static_workspace")
    return out, lse
