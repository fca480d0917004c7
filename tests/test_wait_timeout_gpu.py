"""Failure path of the decode kernel without a GPU fault: with a wait bound of
a few hundred cycles the kernel's waits expire, it records the timeout bit
and exits cleanly; the next decode with the normal bound is correct."""
import pytest

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
