"""mla_decode_noalloc: the decode entry point that allocates nothing.

Some callers cannot allocate device memory themselves (processes that work
inside a fixed budget carved out at start-up and route every later device
allocation through their own pool, or latency-critical paths where
cudaMalloc/cudaFree may synchronise the device).  For them the library keeps
the decode scratch in a built-in device array, and the caller passes only
inputs and outputs.  These tests call that entry point through the C ABI and
check it against mla_decode (caller-provided workspace) on the same inputs,
on two calls in a row with different inputs, since every call shares the
built-in array and it keeps the previous call's contents.

This file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

from mla_latent_kv_25_b200 import binding, inputs
from tests._util import assert_close, to_np


def _noalloc_raw(d, w, out, lse, num_splits):
    """Call the C entry point directly with raw device pointers."""
    lib = binding.load()
    kind = binding.MLA_CACHE_BF16 if d["cache"].dtype == torch.bfloat16 else binding.MLA_CACHE_FP8_E4M3
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.mla_decode_noalloc(P(d["q"]), kind, P(d["cache"]), P(d["k_rope"]),
                                  P(d["block_scale"]), P(d["block_table"]), P(d["seq_lens"]),
                                  w.B, w.H, w.num_blocks, w.max_blocks, float(w.softmax_scale),
                                  P(out), P(lse), int(num_splits), stream)


def test_noalloc_rejects_requests_beyond_its_scratch():
    """A split count whose scratch need exceeds the built-in 40 MiB array is
    rejected on the host (MLA_ERR_WORKSPACE_TOO_SMALL) before any launch."""
    lib = binding.load()
    g = ctypes.c_void_p(4096)
    st = lib.mla_decode_noalloc(g, 0, g, None, None, g, g, 64, 128, 4096, 64, 0.07, g, g,
                                4096, None)
    assert st == 3, binding.STATUS.get(st, st)
    assert binding.mla_decode_workspace_bytes(64, 128, 4096) > (40 << 20)


@pytest.mark.gpu
def test_noalloc_matches_decode_on_two_calls_in_a_row():
    cases = [
        (inputs.make("ragged", B=6, H=128, L=[1, 63, 64, 65, 3000, 130], seed=41, q_std=2.0), 0),
        (inputs.make("v3", B=5, H=64, L=[700, 64, 5, 2000, 129], seed=42, q_std=3.0), 9),
    ]
    for w, splits in cases:
        d = binding.to_device(w)
        ref_out, ref_lse, ws = binding.decode_device(d, w.softmax_scale, num_splits=splits)
        assert binding.mla_get_device_error(ws) == 0
        out = torch.full((w.B, w.H, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((w.B, w.H), float("nan"), dtype=torch.float32, device="cuda")
        st = _noalloc_raw(d, w, out, lse, splits)
        assert st == 0, binding.STATUS.get(st, st)
        torch.cuda.synchronize()
        assert_close(to_np(out).reshape(-1, 512), to_np(ref_out).reshape(-1, 512), "noalloc out")
        assert_close(to_np(lse).reshape(-1), to_np(ref_lse).reshape(-1), "noalloc lse")


@pytest.mark.gpu
def test_noalloc_fp8_beyond_its_room_runs_in_groups():
    """An fp8 batch whose widened copy (16 sequences x 64 blocks x 72 KB =
    75 MB) exceeds the 40 MiB array runs in groups of sequences there and
    matches mla_decode with a whole-batch workspace; the array's error word
    reads 0 afterwards."""
    w = inputs.make("fp8", B=16, H=128, L=4096, seed=48)
    d = binding.to_device(w)
    assert binding.mla_decode_fp8_workspace_bytes(w.B, w.H, w.max_blocks, 0) > (40 << 20)
    ref_out, ref_lse, ws = binding.decode_device(d, w.softmax_scale)
    assert binding.mla_get_device_error(ws) == 0
    out = torch.full((w.B, w.H, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((w.B, w.H), float("nan"), dtype=torch.float32, device="cuda")
    st = _noalloc_raw(d, w, out, lse, 0)
    assert st == 0, binding.STATUS.get(st, st)
    assert binding.mla_decode_noalloc_get_error() == 0
    assert_close(to_np(out).reshape(-1, 512), to_np(ref_out).reshape(-1, 512), "noalloc fp8 groups out")
    assert_close(to_np(lse).reshape(-1), to_np(ref_lse).reshape(-1), "noalloc fp8 groups lse")


@pytest.mark.gpu
def test_noalloc_fp8_cache_matches_decode():
    """An fp8 cache through the built-in scratch: small enough that its
    widened copy fits there, so it takes the tensor-core route as mla_decode
    does with an fp8-sized workspace."""
    w = inputs.make("fp8", B=3, H=32, L=[200, 64, 1], seed=47, q_std=2.0, extra_blocks=2)
    d = binding.to_device(w)
    ref_out, ref_lse, ws = binding.decode_device(d, w.softmax_scale, num_splits=3)
    assert binding.mla_get_device_error(ws) == 0
    out = torch.full((w.B, w.H, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((w.B, w.H), float("nan"), dtype=torch.float32, device="cuda")
    st = _noalloc_raw(d, w, out, lse, 3)
    assert st == 0, binding.STATUS.get(st, st)
    torch.cuda.synchronize()
    assert_close(to_np(out).reshape(-1, 512), to_np(ref_out).reshape(-1, 512), "noalloc fp8 out")
    assert_close(to_np(lse).reshape(-1), to_np(ref_lse).reshape(-1), "noalloc fp8 lse")


@pytest.mark.gpu
def test_noalloc_timeout_after_a_wide_split_call_stays_defined():
    """The built-in scratch keeps the previous call's per-sequence records: a
    call cut over 512 engines (B=1, H=16) leaves records naming high engine
    slots; a following H=128 call whose waits expire must not merge from
    them.  Its rows read out = 0, lse = NaN, the timeout bit is reported by
    mla_decode_noalloc_get_error, and the next call is right again."""
    w1 = inputs.make("v3", B=1, H=16, L=[5000], seed=49)
    d1 = binding.to_device(w1)
    out1 = torch.empty((1, 16, 512), dtype=torch.bfloat16, device="cuda")
    lse1 = torch.empty((1, 16), dtype=torch.float32, device="cuda")
    assert _noalloc_raw(d1, w1, out1, lse1, 512) == 0
    assert binding.mla_decode_noalloc_get_error() == 0
    w2 = inputs.make("v3", B=2, H=128, L=[3000, 700], seed=50)
    d2 = binding.to_device(w2)
    out2 = torch.full((2, 128, 512), 7.0, dtype=torch.bfloat16, device="cuda")
    lse2 = torch.full((2, 128), 7.0, dtype=torch.float32, device="cuda")
    prev = binding.mla_set_wait_limit(1000)
    try:
        st = _noalloc_raw(d2, w2, out2, lse2, 4)
        torch.cuda.synchronize()
    finally:
        binding.mla_set_wait_limit(0)
    assert st == 0, binding.STATUS.get(st, st)
    err = binding.mla_decode_noalloc_get_error()
    assert err & binding.DEVERR_TIMEOUT and not err & binding.DEVERR_BAD_PIECES
    assert torch.all(out2 == 0) and torch.all(torch.isnan(lse2))
    ref_out, ref_lse, ws = binding.decode_device(d2, w2.softmax_scale, num_splits=4)
    assert _noalloc_raw(d2, w2, out2, lse2, 4) == 0
    torch.cuda.synchronize()
    assert binding.mla_decode_noalloc_get_error() == 0
    assert_close(to_np(out2).reshape(-1, 512), to_np(ref_out).reshape(-1, 512), "noalloc after timeout out")
    assert_close(to_np(lse2).reshape(-1), to_np(ref_lse).reshape(-1), "noalloc after timeout lse")
