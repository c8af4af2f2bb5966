"""Failure detection without a GPU fault.

Every wait in the kernels of this library is bounded: after its time limit it
gives up, raises BSA_FLAG_TIMEOUT in the workspace status word, lets the copies
and MMAs already issued drain and returns, so the context stays usable.  On the
GPU this runs the bounded wait itself on a barrier that nothing ever completes
(bsa_selftest_wait_timeout), then checks that a normal call still works.  On the
CPU it checks how the host reports such a status."""
import time

import pytest
import torch

import block_sparse_variable_b200 as bsa
import oracle
import workloads
from tests import harness as H

BSA_FLAG_TIMEOUT = 0x8


def test_status_strings_name_the_failures():
    assert "WORKSPACE" in bsa.bsa_status_string(161004)
    assert bsa.bsa_status_string(0).startswith("BSA_OK")


def test_selftest_rejects_a_null_flag_word():
    with pytest.raises(RuntimeError):
        bsa._check(bsa.lib().bsa_selftest_wait_timeout(None, None), "bsa_selftest_wait_timeout")


@pytest.mark.gpu
def test_bounded_wait_gives_up_and_the_context_stays_usable():
    flags = torch.zeros(16, dtype=torch.int32, device="cuda")
    t0 = time.time()
    bsa.bsa_selftest_wait_timeout(flags)
    torch.cuda.synchronize()
    waited = time.time() - t0
    word = int(flags[0].item()) & 0xFFFFFFFF
    assert word & BSA_FLAG_TIMEOUT, hex(word)
    assert not word & 0x80000000, "the wait returned success on a barrier nobody completed"
    assert 1.0 < waited < 60.0, waited
    # the next call on the same context runs and is correct
    p = workloads.make_config(1)
    d = H.device_inputs(p)
    out, lse, ws, _ = H.gpu_fwd(p, d)
    torch.cuda.synchronize()
    ref_out, ref_lse, _ = oracle.Oracle(p).fwd()
    H.check_close("out", out, ref_out)
    H.check_lse(lse, ref_lse)
    assert bsa.bsa_read_status(ws) == 0
