"""GPU parity: mla_decode / mla_combine / mla_absorb_q through the C ABI
against the FP64 oracle on the same seeded inputs."""
import math

import numpy as np
import pytest
import torch

import oracle
from mla_latent_kv_25_b200 import binding, inputs
from tests._util import assert_close, to_np

pytestmark = pytest.mark.gpu


def run(w, num_splits=0):
    d = binding.to_device(w)
    out, lse, ws = binding.decode_device(d, w.softmax_scale, num_splits=num_splits)
    err = binding.mla_get_device_error(ws)
    return out, lse, err


def check_full(w, num_splits=0, what=""):
    out, lse, err = run(w, num_splits)
    assert err == 0, f"device error bits {err:#x}"
    ro, rl = oracle.decode_workload(w)
    assert_close(to_np(out).reshape(-1, 512), ro, what + " out")
    assert_close(to_np(lse).reshape(-1), rl, what + " lse")
    return out, lse


# ---------------------------------------------------------------- small cases, every element

def test_tiny_config_matches_oracle():
    w = inputs.make("tiny")
    check_full(w, what="tiny")


@pytest.mark.parametrize("num_splits", [0, 1, 2, 3, 7, 64, 200])
def test_ragged_small_all_split_counts(num_splits):
    w = inputs.make("ragged", B=6, H=32, L=[1, 63, 64, 65, 1000, 130], seed=21, q_std=2.0,
                    extra_blocks=4)
    check_full(w, num_splits, what=f"splits={num_splits}")


@pytest.mark.parametrize("H", [16, 48, 128])
def test_head_counts(H):
    w = inputs.make("v3", B=3, H=H, L=[300, 64, 129], seed=22, q_std=1.5)
    check_full(w, what=f"H={H}")


def test_sharp_softmax():
    """Peaked rows (large query spread): errors in the scores show up here."""
    w = inputs.make("v3", B=2, H=64, L=[777, 200], seed=23, q_std=6.0)
    check_full(w, 5, what="sharp")


@pytest.mark.parametrize("route", ["whole", "groups"])
def test_fp8_cache_small(route):
    """The fp8 cache widened for the whole batch at once (workspace sized by
    mla_decode_fp8_workspace_bytes) and one sequence at a time (a workspace
    with room for one sequence's widened copy only)."""
    w = inputs.make("fp8", B=3, H=32, L=[200, 64, 1], seed=24, q_std=2.0, extra_blocks=2)
    d = binding.to_device(w)
    ws = None if route == "whole" else binding.alloc_workspace(1, w.H, 3, fp8_max_blocks=w.max_blocks)
    out, lse, ws = binding.decode_device(d, w.softmax_scale, num_splits=3, workspace=ws)
    assert binding.mla_get_device_error(ws) == 0
    ro, rl = oracle.decode_workload(w)
    assert_close(to_np(out).reshape(-1, 512), ro, f"fp8 {route} out")
    assert_close(to_np(lse).reshape(-1), rl, f"fp8 {route} lse")


def test_fp8_groups_agree_on_a_ragged_batch():
    """Whole-batch widening and groups of two sequences (3 groups, the last
    one short) give the oracle's result; a workspace without room for one
    sequence's widened copy is rejected before any launch."""
    w = inputs.make("fp8", B=5, H=64, L=[1, 700, 65, 64, 2000], seed=33, q_std=3.0, extra_blocks=3)
    d = binding.to_device(w)
    o1, l1, ws1 = binding.decode_device(d, w.softmax_scale, num_splits=4)
    o2, l2, ws2 = binding.decode_device(d, w.softmax_scale, num_splits=4,
                                        workspace=binding.alloc_workspace(2, w.H, 4, fp8_max_blocks=w.max_blocks))
    assert binding.mla_get_device_error(ws1) == 0 and binding.mla_get_device_error(ws2) == 0
    small = binding.alloc_workspace(w.B, w.H, 4)   # split-KV scratch only
    if binding.mla_decode_fp8_workspace_bytes(1, w.H, w.max_blocks, 1) > small.numel():
        with pytest.raises(binding.MLAError) as ei:
            binding.decode_device(d, w.softmax_scale, num_splits=4, workspace=small)
        assert ei.value.status == 3
    ro, rl = oracle.decode_workload(w)
    for o, l, what in ((o1, l1, "whole"), (o2, l2, "groups")):
        assert_close(to_np(o).reshape(-1, 512), ro, f"fp8 {what} out")
        assert_close(to_np(l).reshape(-1), rl, f"fp8 {what} lse")


@pytest.mark.parametrize("cache", ["bf16", "fp8"])
def test_rows_past_seq_len_are_never_used(cache):
    """NaN/huge values in the unused rows of each sequence's last block must
    not reach the output."""
    w = inputs.make("v3", B=3, H=16, L=[70, 130, 5], cache=cache, seed=25, tail_fill=float("nan"))
    check_full(w, 2, what="tail-nan")
    w = inputs.make("v3", B=3, H=16, L=[70, 130, 5], cache=cache, seed=25, tail_fill=3e38)
    check_full(w, 0, what="tail-huge")


def test_empty_sequences():
    w = inputs.make("v3", B=4, H=16, L=[0, 100, 0, 64], seed=26)
    out, lse = check_full(w, 3, what="empty")
    o = to_np(out)
    assert np.all(o[0] == 0) and np.all(o[2] == 0)
    assert np.all(np.isneginf(to_np(lse)[[0, 2]]))


@pytest.mark.parametrize("cache", ["bf16", "fp8"])
@pytest.mark.parametrize("num_splits", [0, 5])
def test_block_relocation_is_bit_exact(cache, num_splits):
    """Physical placement of blocks must not change a single output bit."""
    w = inputs.make("v3", B=3, H=32, L=[500, 64, 129], cache=cache, seed=27, extra_blocks=7)
    w2 = inputs.relocate(w, seed=5)
    o1, l1, e1 = run(w, num_splits)
    o2, l2, e2 = run(w2, num_splits)
    assert e1 == 0 and e2 == 0
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1.view(torch.int32), l2.view(torch.int32))


def test_constant_latent_column():
    """Softmax weights sum to one: a latent column of ones reads back as 1."""
    w = inputs.make("v3", B=2, H=32, L=[1000, 77], seed=28, q_std=3.0)
    w.cache[:, :, 5] = 1.0
    out, lse, err = run(w, 4)
    assert err == 0
    assert np.max(np.abs(to_np(out)[:, :, 5] - 1.0)) <= 2 ** -8


def test_single_token_and_zero_query():
    w = inputs.make("v3", B=2, H=16, L=[1, 64], seed=29)
    w.q[1].zero_()
    out, lse, err = run(w)
    assert err == 0
    row = w.cache[int(w.block_table[0, 0]), 0, :512].float().numpy()
    assert np.max(np.abs(to_np(out)[0] - row[None])) <= 2 ** -8 * np.max(np.abs(row))
    assert np.max(np.abs(to_np(lse)[1] - math.log(64))) < 1e-4


# ---------------------------------------------------------------- device-side checks

@pytest.mark.parametrize("cache", ["bf16", "fp8"])
def test_bad_block_id_sets_error_bit(cache):
    w = inputs.make("v3", B=2, H=16, L=[100, 100], cache=cache, seed=30)
    w.block_table[1, 1] = w.num_blocks + 5
    out, lse, err = run(w)
    assert err & binding.DEVERR_BAD_BLOCK
    # the rows of the other sequence are still right
    ro, rl = oracle.decode_workload(w, rows=np.array([[0, h] for h in range(w.H)], np.int32))
    assert_close(to_np(out)[0], ro, "good sequence next to a bad block")


def test_seq_len_beyond_table_sets_error_bit():
    w = inputs.make("v3", B=2, H=16, L=[100, 100], seed=31)
    w.seq_lens[0] = 64 * w.max_blocks + 1
    out, lse, err = run(w)
    assert err & binding.DEVERR_SEQ_TOO_LONG


# ---------------------------------------------------------------- combine and absorb

def test_combine_matches_oracle():
    g = torch.Generator().manual_seed(32)
    B, H, S = 3, 16, 5
    o = torch.randn((B, H, S, 512), generator=g)
    l = torch.randn((B, H, S), generator=g) * 3
    l[0, 0, :] = -math.inf
    l[1, 2, 1:] = -math.inf
    out = torch.empty((B, H, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
    binding.mla_combine(o.cuda(), l.cuda(), out, lse)
    ro, rl = oracle.combine(o.double().reshape(B * H, S, 512).numpy(), l.double().reshape(B * H, S).numpy())
    assert_close(to_np(out).reshape(-1, 512), ro, "combine out")
    assert_close(to_np(lse).reshape(-1), rl, "combine lse", max_abs=1e-5)


@pytest.mark.parametrize("B,H,ldq", [(1, 16, 576), (5, 32, 576), (64, 128, 576), (130, 16, 640),
                                     (257, 32, 576)])
def test_absorb_q_matches_oracle(B, H, ldq):
    """Tensor-core absorption: several 128-row tiles with a ragged last tile,
    a padded row stride, every head count of the header's range ends."""
    w = inputs.make("v3", B=B, H=H, L=[1] * B, seed=33)
    qn, wu = w.q_nope.cuda(), w.w_uk.cuda()
    qr = w.q[:, :, 512:].contiguous().cuda()
    q_out = torch.full((B, H, ldq), 7.0, dtype=torch.bfloat16, device="cuda")
    binding.mla_absorb_q(qn, wu, qr, q_out)
    assert binding.mla_absorb_get_error() == 0
    ref = oracle.absorb_q(w.q_nope, w.w_uk)
    assert_close(to_np(q_out[:, :, :512]).reshape(-1, 512), ref.reshape(-1, 512), "absorb")
    assert torch.equal(q_out[:, :, 512:576].cpu(), w.q[:, :, 512:])
    assert torch.all(q_out[:, :, 576:] == 7.0)  # padding past the row untouched


def test_absorb_q_without_rope_leaves_tail():
    B, H = 3, 16
    w = inputs.make("v3", B=B, H=H, L=[1] * B, seed=34)
    q_out = torch.full((B, H, 576), 5.0, dtype=torch.bfloat16, device="cuda")
    binding.mla_absorb_q(w.q_nope.cuda(), w.w_uk.cuda(), None, q_out)
    assert binding.mla_absorb_get_error() == 0
    ref = oracle.absorb_q(w.q_nope, w.w_uk)
    assert_close(to_np(q_out[:, :, :512]).reshape(-1, 512), ref.reshape(-1, 512), "absorb no-rope")
    assert torch.all(q_out[:, :, 512:] == 5.0)


@pytest.mark.parametrize("B,H,ldo", [(1, 16, 128), (64, 128, 128), (130, 32, 136)])
def test_absorb_o_matches_oracle(B, H, ldo):
    """Tensor-core output absorption: several 128-row tiles with a ragged last
    tile and a padded row stride."""
    w = inputs.make("v3", B=B, H=H, L=[1] * B, seed=35)
    g = torch.Generator().manual_seed(36)
    o = (torch.randn((B, H, 512), generator=g) * 0.05).to(torch.bfloat16)
    out = torch.full((B, H, ldo), 3.0, dtype=torch.bfloat16, device="cuda")
    binding.mla_absorb_o(o.cuda(), w.w_uv.cuda(), out)
    assert binding.mla_absorb_get_error() == 0
    ref = oracle.absorb_o(o, w.w_uv)
    assert_close(to_np(out[:, :, :128]).reshape(-1, 128), ref.reshape(-1, 128), "absorb_o")
    assert torch.all(out[:, :, 128:] == 3.0)


def test_decode_then_output_absorption_matches_oracle_chain():
    """The layer output of the absorbed path: mla_absorb_q -> mla_decode ->
    mla_absorb_o on the GPU against the oracle's chain on the same inputs."""
    w = inputs.make("v3", B=3, H=32, L=[300, 64, 129], seed=37, q_std=1.0)
    d = binding.to_device(w)
    q = torch.empty((3, 32, 576), dtype=torch.bfloat16, device="cuda")
    binding.mla_absorb_q(d["q_nope"], d["w_uk"], w.q[:, :, 512:].contiguous().cuda(), q)
    d["q"] = q
    out, lse, ws = binding.decode_device(d, w.softmax_scale, num_splits=4)
    assert binding.mla_get_device_error(ws) == 0
    o_heads = torch.empty((3, 32, 128), dtype=torch.bfloat16, device="cuda")
    binding.mla_absorb_o(out, d["w_uv"], o_heads)
    assert binding.mla_absorb_get_error() == 0
    # oracle chain on the same bf16 values the GPU consumed at each step
    w.q = q.cpu()
    ro, _ = oracle.decode_workload(w)
    o_bf = torch.from_numpy(ro.reshape(3, 32, 512)).to(torch.bfloat16)
    ref = oracle.absorb_o(o_bf, w.w_uv)
    assert_close(to_np(o_heads).reshape(-1, 128), ref.reshape(-1, 128), "decode + absorb_o")


def _multi_reference(w, q_len, H):
    """Oracle view of a multi-token decode: token j of sequence b is its own
    sequence sharing b's block table, shorter by q_len - 1 - j tokens."""
    B = w.B
    q = w.q.reshape(B * q_len, H, 576)
    table = w.block_table.repeat_interleave(q_len, dim=0)
    lens = torch.tensor([max(0, int(w.seq_lens[b]) - (q_len - 1 - j)) for b in range(B) for j in range(q_len)],
                        dtype=torch.int32)
    return oracle.decode_units(q=q, cache=w.cache, block_table=table, seq_lens=lens,
                               num_blocks=w.num_blocks, softmax_scale=w.softmax_scale,
                               units=oracle.all_units(B * q_len, H), cache_kind=w.cache_dtype)


@pytest.mark.parametrize("q_len,H,num_splits", [(2, 32, 0), (2, 64, 5), (4, 32, 3), (4, 16, 0),
                                               (2, 128, 0), (4, 128, 5), (4, 64, 4)])
def test_multi_token_decode_matches_oracle(q_len, H, num_splits):
    """q_len query tokens per sequence share the cache pass; token j is causal
    among the drafts (sees all but the last q_len - 1 - j tokens).  Lengths
    include one shorter than q_len (its first tokens see nothing).  Above 128
    rows (H = 128 with 2 and 4 tokens, 4 x 64) the rows run in
    tiles of 128, one cache pass each."""
    B = 4
    w = inputs.make("v3", B=B, H=q_len * H, L=[700, 65, 130, 2], seed=46, q_std=2.0)
    d = binding.to_device(w)
    q = d["q"].reshape(B, q_len, H, 576)
    out = torch.empty((B, q_len, H, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, q_len, H), dtype=torch.float32, device="cuda")
    ws = binding.alloc_workspace(B, q_len * H, num_splits)
    binding.mla_decode_multi(q, d["cache"], d["block_table"], d["seq_lens"], w.softmax_scale, out, lse,
                             ws, num_splits=num_splits)
    assert binding.mla_get_device_error(ws) == 0
    ro, rl = _multi_reference(w, q_len, H)
    assert_close(to_np(out).reshape(-1, 512), ro, f"multi q_len={q_len}")
    finite = np.isfinite(rl)
    assert np.array_equal(np.isfinite(to_np(lse).reshape(-1)), finite)
    assert_close(to_np(lse).reshape(-1)[finite], rl[finite], f"multi lse q_len={q_len}")


# ---------------------------------------------------------------- full-size configs, every row

@pytest.mark.parametrize("name", ["v3", "ragged", "long", "fp8"])
def test_full_config_every_row(name):
    """Every output row and lse of each full-size workload, in the launch
    configuration the benchmark times (automatic split count), against the
    oracle computed for the whole workload (multithreaded fp64 C: a few
    seconds to tens of seconds per workload on the host cores)."""
    w = inputs.make(name)
    out, lse, err = run(w)
    assert err == 0
    ro, rl = oracle.decode_workload(w)
    assert_close(to_np(out).reshape(-1, 512), ro, name + " out")
    assert_close(to_np(lse).reshape(-1), rl, name + " lse")


# ---------------------------------------------------------------- determinism under load

@pytest.mark.parametrize("num_splits", [3, 5, 6])
def test_repeated_runs_are_bit_identical(num_splits):
    """Engines that hold several sequence pieces (short first segment, then
    another sequence) hand the output accumulator between warps at segment
    ends; every repeat of the same call must give identical bits and stay
    within tolerance of the oracle."""
    w = inputs.make("v3", B=4, H=128, L=[700, 300, 64, 900], seed=5, q_std=3.0)
    d = binding.to_device(w)
    ref_out = ref_lse = None
    ro, rl = oracle.decode_workload(w)
    for rep in range(12):
        out, lse, ws = binding.decode_device(d, w.softmax_scale, num_splits=num_splits)
        assert binding.mla_get_device_error(ws) == 0
        if ref_out is None:
            ref_out, ref_lse = out.clone(), lse.clone()
            assert_close(to_np(out).reshape(-1, 512), ro, "repeat out")
            assert_close(to_np(lse).reshape(-1), rl, "repeat lse")
        else:
            assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16)), f"repeat {rep}"
            assert torch.equal(lse.view(torch.int32), ref_lse.view(torch.int32)), f"repeat {rep}"
