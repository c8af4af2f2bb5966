"""The paired fp32 operations of the backward kernels' softmax (csrc/f32x2.cuh:
fma/add/mul .rn.f32x2, two elements per instruction) give the same bits as the
scalar round-to-nearest operations, through bsa_selftest_f32x2.  The softmax
relies on it: its P and dS are meant to be those of the scalar arithmetic."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def _same_bits(x, y):
    """Bitwise equality, any NaN equal to any NaN."""
    nan = torch.isnan(x) & torch.isnan(y)
    return bool(((x.view(torch.int32) == y.view(torch.int32)) | nan).all())


def test_paired_equals_scalar():
    import block_sparse_variable_b200 as bsa
    g = torch.Generator().manual_seed(7)
    n = 1 << 20
    a = torch.randn(n, generator=g) * 8
    b = torch.randn(n, generator=g) * 8
    c = torch.randn(n, generator=g) * 64
    # the softmax's own ranges: scores times scale*log2(e) minus lse, and
    # values near cancellation, denormals, zeros of both signs, infinities
    special = torch.tensor([0.0, -0.0, 1e-40, -1e-40, 3e38, -3e38, float("inf"), float("-inf"),
                            float("nan"), 1.0, -1.0, 0.5, 2.0 ** -126, 2.0 ** -149, 1 + 2.0 ** -23,
                            1 - 2.0 ** -24])
    k = special.numel()
    a[:k * k] = special.repeat_interleave(k)
    b[:k * k] = special.repeat(k)
    c[:k * k] = -a[:k * k] * b[:k * k]
    a, b, c = (t.cuda() for t in (a, b, c))
    pair, scal = bsa.bsa_selftest_f32x2(a, b, c)
    torch.cuda.synchronize()
    for row, name in enumerate(("fma", "add", "mul")):
        assert _same_bits(pair[row], scal[row]), name
    # and both are the IEEE results torch computes for add and mul
    assert _same_bits(scal[1], a + b)
    assert _same_bits(scal[2], a * b)


def test_rejects_odd_or_negative_n():
    import block_sparse_variable_b200 as bsa
    lib = bsa.lib()
    x = torch.zeros(4, device="cuda")
    p = x.data_ptr()
    assert lib.bsa_selftest_f32x2(p, p, p, p, p, 3, None) != 0
    assert lib.bsa_selftest_f32x2(p, p, p, p, p, -2, None) != 0
    assert lib.bsa_selftest_f32x2(None, p, p, p, p, 2, None) != 0
    assert lib.bsa_selftest_f32x2(p, p, p, p, p, 0, None) == 0
