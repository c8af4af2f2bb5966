"""The C-ABI library without a GPU: it loads, exports every entry point the
header declares, and its host-side validation and workspace sizing behave
(these paths never touch device memory, so host tensors stand in)."""
import os
import re

import pytest
import torch

import block_sparse_variable_b200 as bsa
from workloads.gen import make_problem, pat_random_k
from tests.harness import params_of

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "bsa.h")).read()
    return sorted(set(re.findall(r"^\s*(?:bsa_status|const char \*|int32_t)\s*(bsa_\w+)\(", src, re.M)))


def test_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 9
    for n in names:
        assert hasattr(bsa.lib(), n), n
    assert set(names) == set(bsa.EXPORTED)
    assert bsa.lib().bsa_abi_version() == 3


def test_status_strings():
    for code, name in bsa.STATUS_NAMES.items():
        assert bsa.bsa_status_string(code).startswith(name)


def _prob(**kw):
    base = dict(layout_q="TND", layout_kv="TND", B=2, N1=4, N2=2, D=64, lens_q=[200, 130],
                pattern=pat_random_k, seed_base=1)
    base.update(kw)
    return make_problem(**base)


def _ws(p, params=None, **over):
    a = dict(q=p.q, k=p.k, v=p.v, index=p.index, cu_seqlens_q=p.cu_q, cu_seqlens_kv=p.cu_kv,
             seqused_kv=p.seqused_kv, block_table=p.block_table)
    a.update(over)
    return bsa.bsa_fwd_get_workspace(a.pop("q"), a.pop("k"), a.pop("v"), a.pop("index"),
                                     params or params_of(p), **a)


def _code(fn):
    with pytest.raises(bsa.BsaError) as e:
        fn()
    return e.value.status


def test_valid_layouts_size_workspace():
    for kw in (dict(), dict(layout_q="BNSD", layout_kv="BNSD", Sq=300, lens_q=None, lens_kv=None),
               dict(layout_kv="PA_BBND", page_size=256)):
        p = _prob(**kw)
        n = _ws(p)
        lay = bsa.bsa_fwd_workspace_layout(p.q, p.k, p.v, p.index, params_of(p), cu_seqlens_q=p.cu_q,
                                           cu_seqlens_kv=p.cu_kv, seqused_kv=p.seqused_kv,
                                           block_table=p.block_table,
                                           lse=torch.empty(p.q.shape[:-1] if p.layout_q == "TND"
                                                           else p.q.shape[:-1], dtype=torch.float32))
        assert n == lay.total_bytes > 0
        regs = sorted((getattr(lay, f).offset, getattr(lay, f).bytes) for f in
                      ("status", "batch", "comp", "ncomp", "fwd_items", "sort_keys")
                      if getattr(lay, f).bytes)
        for (o1, b1), (o2, _) in zip(regs, regs[1:]):
            assert o1 + b1 <= o2 and o1 % 256 == 0
        assert regs[-1][0] + regs[-1][1] <= n
        assert lay.status.offset == 0


def test_backward_workspace_has_inverse_and_accumulator():
    p = _prob()
    lse = torch.empty(p.q.shape[0], p.N1)
    lay = bsa.bsa_bwd_workspace_layout(p.q, p.k, p.v, p.q, p.dout, lse, p.index, params_of(p),
                                       cu_seqlens_q=p.cu_q, cu_seqlens_kv=p.cu_kv)
    assert lay.inv_off.bytes and lay.inv_list.bytes and lay.bwd_items.bytes
    assert lay.dq_acc.bytes == p.q.shape[0] * p.N1 * p.D * 4
    assert lay.dsum.bytes == p.q.shape[0] * p.N1 * 4
    n = bsa.bsa_bwd_get_workspace(p.q, p.k, p.v, p.q, p.dout, lse, p.index, params_of(p),
                                  cu_seqlens_q=p.cu_q, cu_seqlens_kv=p.cu_kv)
    assert n == lay.total_bytes


def test_rejections():
    p = _prob()
    P = params_of(p)
    ok = _ws(p)
    assert ok > 0
    # missing required pieces
    assert _code(lambda: bsa.bsa_fwd_get_workspace(p.q, p.k, p.v, p.index, P, cu_seqlens_kv=p.cu_kv)) \
        == 161001
    assert _code(lambda: _ws(p, cu_seqlens_kv=None)) == 161001
    # shapes / dtypes / attributes
    assert _code(lambda: _ws(p, k=p.k.float())) == 161002
    assert _code(lambda: _ws(p, params=bsa.params_for("TND", "TND", 4, 3, (128, 128)))) == 161002
    assert _code(lambda: _ws(p, params=bsa.params_for("TND", "TND", 4, 2, (64, 128)))) == 161002
    assert _code(lambda: _ws(p, params=bsa.params_for("TND", "TND", 4, 2, (128, 2048)))) == 161002
    assert _code(lambda: _ws(p, params=bsa.params_for("TND", "BNSD", 4, 2, (128, 128)))) == 161002
    assert _code(lambda: _ws(p, params=bsa.params_for("TND", "TND", 5, 2, (128, 128)))) == 161002
    assert _code(lambda: _ws(p, params=bsa.params_for("TND", "TND", 4, 2, (128, 128), scale=-1.0))) \
        == 161002
    assert _code(lambda: _ws(p, index=p.index.view(torch.int16))) == 161002
    assert _code(lambda: _ws(p, index=p.index[:3])) == 161002          # Hidx not N1 / N2
    assert _code(lambda: _ws(p, q=p.q[:, :, :48].contiguous(), k=p.k[:, :, :48].contiguous(),
                             v=p.v[:, :, :48].contiguous())) == 161003   # D = 48
    # strides: last dim contiguous, others 16-byte multiples
    strided = torch.zeros(p.q.shape[0], p.q.shape[1], 128, dtype=p.q.dtype)[..., ::2]
    assert _code(lambda: _ws(p, q=strided)) == 161002
    wide = torch.zeros(p.q.shape[0], p.q.shape[1], 68, dtype=p.q.dtype)[..., :64]  # row stride 68
    assert _code(lambda: _ws(p, q=wide)) == 161002
    # paged: page size multiple of 128; seqused required
    pp = _prob(layout_kv="PA_BBND", page_size=128)
    assert _ws(pp) > 0
    assert _code(lambda: _ws(pp, seqused_kv=None)) == 161001
    assert _code(lambda: _ws(pp, cu_seqlens_kv=torch.zeros(3, dtype=torch.int64))) == 161002
    p64 = _prob(layout_kv="PA_BBND", page_size=64)
    assert _code(lambda: _ws(p64)) == 161003


def test_bnsd_index_shape_and_lse():
    p = _prob(layout_q="BNSD", layout_kv="BNSD", Sq=300, lens_q=None, lens_kv=None)
    assert _ws(p) > 0
    assert _code(lambda: _ws(p, index=p.index[:, :, :2])) == 161002     # rows != ceil(S/BQ)
    P = params_of(p)
    bad_lse = torch.empty(1, 4, 300)
    assert _code(lambda: bsa.bsa_fwd_get_workspace(p.q, p.k, p.v, p.index, P, lse=bad_lse)) == 161002


def test_exec_rejects_small_workspace_before_any_launch():
    p = _prob()
    n = _ws(p)
    ws = torch.zeros(n // 2, dtype=torch.uint8)
    with pytest.raises(bsa.BsaError) as e:
        bsa.bsa_fwd(p.q, p.k, p.v, p.index, params_of(p), cu_seqlens_q=p.cu_q,
                    cu_seqlens_kv=p.cu_kv, out=torch.empty_like(p.q),
                    lse=torch.empty(p.q.shape[0], p.N1), workspace=ws, stream=0)
    assert e.value.status == 161004


def test_empty_query_is_a_no_op():
    p = _prob()
    q0 = p.q[:0]
    cu = torch.zeros(3, dtype=torch.int64)
    out, lse, _ = bsa.bsa_fwd(q0, p.k, p.v, p.index[:, :0], params_of(p), cu_seqlens_q=cu,
                              cu_seqlens_kv=p.cu_kv, out=torch.empty_like(q0),
                              lse=torch.empty(0, p.N1), workspace=torch.zeros(256, dtype=torch.uint8),
                              stream=0)
    assert out.numel() == 0


def test_mask_type_must_be_known():
    """bsa_params.mask_type is BSA_MASK_NONE (0) or BSA_MASK_CAUSAL (1)."""
    import dataclasses
    p = _prob()
    P = params_of(p)

    class Bad(bsa.Params):
        def c(self):
            c = super().c()
            c.mask_type = 7
            return c

    bad = Bad(**{f.name: getattr(P, f.name) for f in dataclasses.fields(P)})
    assert _code(lambda: _ws(p, params=bad)) == 161002
    assert _ws(p, params=dataclasses.replace(P, causal=True)) == _ws(p)


def test_deterministic_backward_workspace():
    """The deterministic backward holds the forward work list and no dQ
    accumulator; the forward ignores the flag."""
    import dataclasses
    p = _prob()
    P = params_of(p)
    Pd = dataclasses.replace(P, deterministic=True)
    lse = torch.empty(p.q.shape[0], p.N1)
    kw = dict(cu_seqlens_q=p.cu_q, cu_seqlens_kv=p.cu_kv)
    lay = bsa.bsa_bwd_workspace_layout(p.q, p.k, p.v, p.q, p.dout, lse, p.index, P, **kw)
    lay_d = bsa.bsa_bwd_workspace_layout(p.q, p.k, p.v, p.q, p.dout, lse, p.index, Pd, **kw)
    assert lay.dq_acc.bytes and not lay.fwd_items.bytes
    assert lay_d.fwd_items.bytes and not lay_d.dq_acc.bytes
    assert lay_d.sort_keys.bytes >= lay.sort_keys.bytes
    assert bsa.bsa_bwd_get_workspace(p.q, p.k, p.v, p.q, p.dout, lse, p.index, Pd, **kw) \
        == lay_d.total_bytes
    assert _ws(p, params=Pd) == _ws(p)


def test_fp8_inputs_forward_only():
    """e4m3 q/k/v: out must be f16/bf16 (its dtype is the output type), D must
    be 128, strides 16-byte multiples; the backward refuses them."""
    p = _prob(D=128, dtype=torch.float8_e4m3fn)
    P = params_of(p)
    kw = dict(cu_seqlens_q=p.cu_q, cu_seqlens_kv=p.cu_kv)
    out_bf = torch.empty(p.q.shape, dtype=torch.bfloat16)
    out_h = torch.empty(p.q.shape, dtype=torch.float16)
    lse = torch.empty(p.q.shape[0], p.N1)
    n = bsa.bsa_fwd_get_workspace(p.q, p.k, p.v, p.index, P, out=out_bf, lse=lse, **kw)
    assert n > 0
    assert bsa.bsa_fwd_get_workspace(p.q, p.k, p.v, p.index, P, out=out_h, lse=lse, **kw) == n
    fp8_out = torch.empty(p.q.shape, dtype=torch.float8_e4m3fn)
    assert _code(lambda: bsa.bsa_fwd_get_workspace(p.q, p.k, p.v, p.index, P, out=fp8_out, lse=lse,
                                                   **kw)) == 161002
    assert _code(lambda: bsa.bsa_fwd_get_workspace(p.q, p.k.to(torch.bfloat16), p.v, p.index, P,
                                                   out=out_bf, lse=lse, **kw)) == 161002
    p64 = _prob(D=64, dtype=torch.float8_e4m3fn)
    assert _code(lambda: bsa.bsa_fwd_get_workspace(
        p64.q, p64.k, p64.v, p64.index, params_of(p64),
        out=torch.empty(p64.q.shape, dtype=torch.bfloat16), lse=lse,
        cu_seqlens_q=p64.cu_q, cu_seqlens_kv=p64.cu_kv)) == 161003
    wide = torch.zeros(p.q.shape[0], p.q.shape[1], 136, dtype=torch.float8_e4m3fn)[..., :128]
    assert _code(lambda: bsa.bsa_fwd_get_workspace(wide, p.k, p.v, p.index, P, out=out_bf, lse=lse,
                                                   **kw)) == 161002       # row stride 136
    with pytest.raises(bsa.BsaError) as e:
        bsa.bsa_bwd_get_workspace(p.q, p.k, p.v, out_bf, out_bf, lse, p.index, P, **kw)
    assert e.value.status == 161003


def test_plain_c_caller():
    """A C program built against include/bsa.h alone links libbsa.so and
    sizes workspaces / gets the host refusals (tests/c_abi_check.c)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    pkg = os.path.dirname(bsa.LIB_PATH)
    out_dir = os.path.join(pkg, "_build")
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "c_abi_check")
    subprocess.check_call([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "c_abi_check.c"), "-o", exe,
                           f"-L{pkg}", "-l:libbsa.so", f"-Wl,-rpath,{pkg}"])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"


def test_binding_refuses_to_import_without_the_library():
    """No fallback: a copy of the binding with no libbsa.so beside it raises
    ImportError at import (run in a child process)."""
    import shutil
    import subprocess
    import sys
    pkg = os.path.dirname(bsa.LIB_PATH)
    root = os.path.join(pkg, "_build", "nolib")
    shutil.rmtree(root, ignore_errors=True)
    os.makedirs(os.path.join(root, "block_sparse_variable_b200"))
    shutil.copy(os.path.join(pkg, "__init__.py"), os.path.join(root, "block_sparse_variable_b200"))
    r = subprocess.run([sys.executable, "-c", "import block_sparse_variable_b200"], cwd=root,
                       capture_output=True, text=True, timeout=300,
                       env=dict(os.environ, PYTHONPATH=root))
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "libbsa.so is missing" in r.stderr
