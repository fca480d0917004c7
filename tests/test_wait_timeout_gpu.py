"""Failure path of the decode kernel without a GPU fault: with a wait bound of
a few hundred cycles the kernel's waits expire, it records the timeout bit
and exits cleanly; the next decode with the normal bound is correct."""
import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_25_b200 import binding, inputs
from tests._util import assert_close, to_np

pytestmark = pytest.mark.gpu


def test_expired_waits_report_timeout_and_leave_the_context_usable():
    w = inputs.make("v3", B=3, H=32, L=[700, 64, 129], seed=45)
    d = binding.to_device(w)
    prev = binding.mla_set_wait_limit(1000)
    try:
        out, lse, ws = binding.decode_device(d, w.softmax_scale, num_splits=4)
        err = binding.mla_get_device_error(ws)
    finally:
        binding.mla_set_wait_limit(0)
    assert err & binding.DEVERR_TIMEOUT
    assert prev > 1000
    # the same inputs again, normal bound: correct results, no error
    out, lse, ws = binding.decode_device(d, w.softmax_scale, num_splits=4)
    assert binding.mla_get_device_error(ws) == 0
    ro, rl = oracle.decode_workload(w)
    assert_close(to_np(out).reshape(-1, 512), ro, "after timeout")
    assert_close(to_np(lse).reshape(-1), rl, "after timeout lse")


@pytest.mark.parametrize("H", [16, 128])
def test_timeout_leaves_defined_rows_until_the_error_is_read(H):
    """One sequence cut over every engine (num_splits = 512): with the wait
    bound at 1000 cycles the decode gives up, and the merge reads no piece of
    the incomplete call: every row is 0 with lse = NaN.  The timeout bit is
    sticky: a second call before it is read still gives NaN rows; once
    mla_get_device_error has read (and cleared) it, the same call is right."""
    w = inputs.make("v3", B=1, H=H, L=[5000], seed=46)
    d = binding.to_device(w)
    ws = binding.alloc_workspace(w.B, w.H, 512)
    prev = binding.mla_set_wait_limit(1000)
    try:
        out, lse, _ = binding.decode_device(d, w.softmax_scale, num_splits=512, workspace=ws)
        torch.cuda.synchronize()
        o1, l1 = to_np(out), to_np(lse)
    finally:
        binding.mla_set_wait_limit(0)
    out, lse, _ = binding.decode_device(d, w.softmax_scale, num_splits=512, workspace=ws)
    torch.cuda.synchronize()
    o2, l2 = to_np(out), to_np(lse)
    err = binding.mla_get_device_error(ws)
    assert err & binding.DEVERR_TIMEOUT
    assert not err & binding.DEVERR_BAD_PIECES
    for o, l in ((o1, l1), (o2, l2)):
        assert np.all(o == 0) and np.all(np.isnan(l))
    out, lse, _ = binding.decode_device(d, w.softmax_scale, num_splits=512, workspace=ws)
    assert binding.mla_get_device_error(ws) == 0
    ro, rl = oracle.decode_workload(w)
    assert_close(to_np(out).reshape(-1, 512), ro, "after the error was read")
    assert_close(to_np(lse).reshape(-1), rl, "after the error was read lse")
