"""bsa_fwd_static_workspace: the forward for callers that cannot allocate
device memory while they run (for example a plugin inside an inference
runtime that forbids allocation in its execute step, or an engine whose
memory budget is fixed at start-up).  It uses the library's built-in 32 MiB
scratch array instead of a caller workspace.

This file is collected last on purpose: the test must pass in a fresh
process and after every other test has used the library."""
import ctypes

import pytest
import torch

import block_sparse_variable_b200 as bsa
import workloads
from tests import harness as H


def _call_static(p, d, out, lse):
    # straight through the C ABI
    f = bsa.lib().bsa_fwd_static_workspace
    T = ctypes.POINTER(bsa.bsa_tensor)
    f.argtypes = [T] * 8 + [ctypes.POINTER(bsa.bsa_params), T, T, ctypes.c_void_p]
    f.restype = ctypes.c_int
    descs = [bsa.describe(x) for x in (d["q"], d["k"], d["v"], d["index"], d["cu_seqlens_q"],
                                       d["cu_seqlens_kv"], d["seqused_kv"], d["block_table"])]
    cp = bsa.params_of_problem(p).c()
    st = f(*[None if x is None else ctypes.byref(x) for x in descs], ctypes.byref(cp),
           ctypes.byref(bsa.describe(out)), ctypes.byref(bsa.describe(lse)),
           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


@pytest.mark.gpu
@pytest.mark.parametrize("c", [1, 2, 5])
def test_static_workspace_forward_matches_bsa_fwd(c):
    """Two calls in a row agree with bsa_fwd (same tolerance as the parity
    tests), and once the first call on the device has set the scratch array
    up, a further call leaves the device's free memory unchanged."""
    p = workloads.make_config(c)
    d = H.device_inputs(p)
    ref_out, ref_lse, _, _ = H.gpu_fwd(p, d)
    torch.cuda.synchronize()
    out = torch.empty_like(ref_out)
    lse = torch.empty_like(ref_lse)
    for _ in range(2):
        out.fill_(float("nan"))
        lse.fill_(float("nan"))
        assert _call_static(p, d, out, lse) == 0
        torch.cuda.synchronize()
        H.check_close("out", out, ref_out.double())
        H.check_lse(lse, ref_lse)
    free_before = torch.cuda.mem_get_info()[0]
    assert _call_static(p, d, out, lse) == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before


@pytest.mark.gpu
def test_static_workspace_refusal_clears_armed_events():
    """A pair of events armed for the next call is used up by a refused call
    too: the next bsa_fwd must not record it."""
    p = workloads.make_config(1)
    d = H.device_inputs(p)
    big = _oversized()
    # the pair first spans a ~20 ms sleep; had the refused call left it armed,
    # the next bsa_fwd would record it again around its ~15 us main kernel
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    torch.cuda._sleep(40_000_000)
    e1.record()
    torch.cuda.synchronize()
    assert e0.elapsed_time(e1) > 10.0
    lib = bsa.lib()
    lib.bsa_set_main_kernel_events.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    lib.bsa_set_main_kernel_events.restype = ctypes.c_int
    assert lib.bsa_set_main_kernel_events(ctypes.c_void_p(e0.cuda_event),
                                          ctypes.c_void_p(e1.cuda_event)) == 0
    assert _call_raw(*big) == 161004
    H.gpu_fwd(p, d)
    torch.cuda.synchronize()
    assert e0.elapsed_time(e1) > 10.0


def _oversized():
    """Descriptors of a forward whose workspace exceeds the 32 MiB scratch
    (491 MB of compacted index rows); nothing is read through them."""
    q = bsa.describe_shape((4096, 32, 128), torch.bfloat16)
    k = bsa.describe_shape((4096, 8, 128), torch.bfloat16)
    index = bsa.describe_shape((32, 120000, 64), torch.uint16)
    cu = bsa.describe_shape((2,), torch.int64)
    out = bsa.describe_shape((4096, 32, 128), torch.bfloat16)
    lse = bsa.describe_shape((4096, 32), torch.float32)
    cp = bsa.params_for("TND", "TND", 32, 8).c()
    return q, k, index, cu, out, lse, cp


def _call_raw(q, k, index, cu, out, lse, cp):
    f = bsa.lib().bsa_fwd_static_workspace
    T = ctypes.POINTER(bsa.bsa_tensor)
    f.argtypes = [T] * 8 + [ctypes.POINTER(bsa.bsa_params), T, T, ctypes.c_void_p]
    f.restype = ctypes.c_int
    r = ctypes.byref
    return f(r(q), r(k), r(k), r(index), r(cu), r(cu), None, None, r(cp), r(out), r(lse), None)


def test_static_workspace_rejects_oversized_problems():
    """A forward needing more than the 32 MiB scratch is refused before any
    launch (host-side check only, so no GPU is needed)."""
    assert _call_raw(*_oversized()) == 161004   # BSA_ERR_WORKSPACE
