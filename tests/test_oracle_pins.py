"""Pins for the FP64 oracle: each test checks it against something other than
itself (the unabsorbed textbook form, a library attention routine, closed
forms, invariants, brute-force decoding of the number formats).  CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import naive
from mla_latent_kv_25_b200 import inputs, layout

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- number formats

def test_e4m3_decoder_all_256_codes_match_library():
    """OCP E4M3: all 256 codes against torch's float8_e4m3fn conversion."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    lib_vals = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        v = oracle.e4m3_to_f64(c)
        if math.isnan(lib_vals[c]):
            assert math.isnan(v), c
        else:
            assert v == lib_vals[c], (c, v, lib_vals[c])
            assert math.copysign(1.0, v) == math.copysign(1.0, lib_vals[c])


def test_e4m3_decoder_spec_values():
    """Values fixed by the OCP FP8 definition (bias 7, 3 mantissa bits)."""
    assert oracle.e4m3_to_f64(0x7E) == 448.0          # largest finite
    assert oracle.e4m3_to_f64(0xFE) == -448.0
    assert oracle.e4m3_to_f64(0x01) == 2.0 ** -9      # smallest subnormal
    assert oracle.e4m3_to_f64(0x07) == 7 * 2.0 ** -9  # largest subnormal
    assert oracle.e4m3_to_f64(0x08) == 2.0 ** -6      # smallest normal
    assert oracle.e4m3_to_f64(0x38) == 1.0
    assert oracle.e4m3_to_f64(0x39) == 1.125
    assert math.isnan(oracle.e4m3_to_f64(0x7F)) and math.isnan(oracle.e4m3_to_f64(0xFF))
    assert oracle.e4m3_to_f64(0x80) == 0.0 and math.copysign(1, oracle.e4m3_to_f64(0x80)) < 0


def test_bf16_decoder_matches_library():
    g = torch.Generator().manual_seed(7)
    bits = torch.randint(0, 1 << 16, (20000,), generator=g, dtype=torch.int32)
    vals = bits.to(torch.int16).view(torch.bfloat16).to(torch.float64).numpy()
    for b, v in zip(bits.tolist(), vals.tolist()):
        o = oracle.bf16_to_f64(b)
        if math.isnan(v):
            assert math.isnan(o)
        else:
            assert o == v
    assert oracle.bf16_to_f64(0x3F80) == 1.0
    assert oracle.bf16_to_f64(0xC000) == -2.0
    assert oracle.bf16_to_f64(0x7F80) == math.inf


# ---------------------------------------------------------------- absorbed == naive

def _paged_f64(rows: np.ndarray, seed: int, extra: int = 2):
    """Place logical rows [L,576] into a randomly permuted f64 paged cache."""
    L = rows.shape[0]
    nblk = (L + 63) // 64
    NB = nblk + extra
    rng = np.random.default_rng(seed)
    perm = rng.permutation(NB)
    cache = rng.standard_normal((NB, 64, 576)) * 100.0   # junk everywhere else
    table = np.full((1, nblk), -1, np.int32)
    for j in range(nblk):
        table[0, j] = perm[j]
        n = min(64, L - 64 * j)
        cache[perm[j], :n] = rows[64 * j: 64 * j + n]
    return cache, table, NB


@pytest.mark.parametrize("L", [256, 1, 63, 65, 200])
def test_absorbed_equals_naive_unabsorbed_form(L):
    """Empirical Gains (priorstack.com): absorbing W_UK into the query and
    W_UV into the output gives exactly the attention of the unabsorbed form.
    FP64 agreement to 1e-10 on the tiny DeepSeek shape (H=16, d_c=512)."""
    H = 16
    raw = inputs.raw_tiny_fp32(seed=0, H=H, L=max(L, 1))
    raw = {k: v.double().numpy() for k, v in raw.items()}
    scale = 1.0 / math.sqrt(192)
    q_pos = L - 1
    o_naive, s_naive = naive.naive_mha(raw["c_kv"], raw["k_r"], raw["q_nope"], raw["q_r"],
                                       raw["w_uk"], raw["w_uv"], scale, q_pos=q_pos)
    # absorbed: cache rows [c_kv | RoPE(k_r)], query [q_nope W_UK | RoPE(q_r)]
    k_rot = naive.rope(raw["k_r"], np.arange(L))
    rows = np.concatenate([raw["c_kv"], k_rot], axis=1)
    cache, table, NB = _paged_f64(rows, seed=L)
    q_abs = np.einsum("hd,hdc->hc", raw["q_nope"], raw["w_uk"])
    q_rot = naive.rope(raw["q_r"], np.full(H, q_pos))
    q = np.concatenate([q_abs, q_rot], axis=1)[None]       # [1,H,576]
    units = oracle.all_units(1, H)
    o_lat, lse = oracle.decode_units(q=q, q_kind="f64", cache=cache, cache_kind="f64",
                                     block_table=table, seq_lens=np.array([L], np.int32),
                                     num_blocks=NB, softmax_scale=scale, units=units)
    o_abs = np.einsum("hdc,hc->hd", raw["w_uv"], o_lat)
    assert np.max(np.abs(o_abs - o_naive)) < 1e-10
    from scipy.special import logsumexp
    assert np.max(np.abs(lse - logsumexp(s_naive, axis=1))) < 1e-10


def test_rope_relative_position_property():
    """RoPE scores depend only on the query-key distance (eeumee.net,
    "Residual & RoPE Explanation"): shifting every position by the same
    offset leaves the naive scores unchanged; rotation keeps norms; position
    0 is the identity."""
    raw = inputs.raw_tiny_fp32(seed=3, H=4, L=40)
    raw = {k: v.double().numpy() for k, v in raw.items()}
    s = 1 / math.sqrt(192)
    _, s0 = naive.naive_mha(raw["c_kv"], raw["k_r"], raw["q_nope"], raw["q_r"], raw["w_uk"],
                            raw["w_uv"], s, q_pos=39, k_pos0=0)
    _, s1 = naive.naive_mha(raw["c_kv"], raw["k_r"], raw["q_nope"], raw["q_r"], raw["w_uk"],
                            raw["w_uv"], s, q_pos=39 + 1234, k_pos0=1234)
    assert np.max(np.abs(s0 - s1)) < 1e-12
    _, s2 = naive.naive_mha(raw["c_kv"], raw["k_r"], raw["q_nope"], raw["q_r"], raw["w_uk"],
                            raw["w_uv"], s, q_pos=39 + 5, k_pos0=0)
    assert np.max(np.abs(s0 - s2)) > 1e-6          # the position does matter
    x = raw["k_r"]
    r = naive.rope(x, np.arange(40) * 7)
    assert np.allclose(np.linalg.norm(r, axis=1), np.linalg.norm(x, axis=1), rtol=0, atol=1e-13)
    assert np.array_equal(naive.rope(x, np.zeros(40)), x)


# ---------------------------------------------------------------- library attention

def _gather_logical(w, b):
    """Logical rows [L,576] of batch row b, decoded with torch (library)."""
    L = int(w.seq_lens[b])
    out = []
    for t in range(L):
        blk = int(w.block_table[b, t // 64])
        r = t % 64
        if w.cache_dtype == "bf16":
            out.append(w.cache[blk, r].double())
        else:
            ck = w.cache[blk, r].view(torch.float8_e4m3fn).double() * float(w.block_scale[blk])
            out.append(torch.cat([ck, w.k_rope[blk, r].double()]))
    if not out:
        return torch.zeros((0, 576), dtype=torch.float64)
    return torch.stack(out)


@pytest.mark.parametrize("cache", ["bf16", "fp8"])
def test_oracle_matches_library_sdpa(cache):
    """Decode attention is plain scaled-dot-product attention over the cached
    rows (values = the latent part); compare with torch's SDPA in fp64 and
    lse with torch.logsumexp."""
    w = inputs.make("v3", B=3, H=16, L=[130, 64, 7], cache=cache, seed=11, q_std=2.0,
                    extra_blocks=3)
    out, lse = oracle.decode_workload(w)
    out = out.reshape(w.B, w.H, 512)
    lse = lse.reshape(w.B, w.H)
    for b in range(w.B):
        K = _gather_logical(w, b)                      # [L,576]
        V = K[:, :512]
        q = w.q[b].double()                            # [H,576]
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[None, :, None, :], K[None, None].expand(1, w.H, -1, -1),
            V[None, None].expand(1, w.H, -1, -1), scale=w.softmax_scale)[0, :, 0]
        assert np.max(np.abs(out[b] - ref.numpy())) < 1e-12
        s = (q @ K.T) * w.softmax_scale
        assert np.max(np.abs(lse[b] - torch.logsumexp(s, dim=1).numpy())) < 1e-12


# ---------------------------------------------------------------- closed forms

def test_single_token_returns_that_row():
    w = inputs.make("v3", B=2, H=8, L=[1, 1], seed=5)
    out, lse = oracle.decode_workload(w)
    for b in range(2):
        row = w.cache[int(w.block_table[b, 0]), 0].double().numpy()
        for h in range(8):
            i = b * 8 + h
            assert np.array_equal(out[i], row[:512])
            s = float(np.dot(w.q[b, h].double().numpy(), row)) * w.softmax_scale
            assert abs(lse[i] - s) < 1e-12


def test_zero_query_gives_mean_and_log_length():
    w = inputs.make("v3", B=2, H=4, L=[100, 257], seed=6)
    w.q.zero_()
    out, lse = oracle.decode_workload(w)
    for b in range(2):
        K = _gather_logical(w, b).numpy()
        for h in range(4):
            i = b * 4 + h
            assert np.max(np.abs(out[i] - K[:, :512].mean(axis=0))) < 1e-14
            assert abs(lse[i] - math.log(K.shape[0])) < 1e-12


def test_constant_latent_column_is_reproduced():
    """Softmax weights sum to one: a latent column equal to 1 in every token
    comes out as exactly 1 for every head."""
    w = inputs.make("v3", B=2, H=8, L=[300, 64], seed=8, q_std=3.0)
    w.cache[:, :, 17] = 1.0
    w.cache[:, :, 400] = -2.0
    out, _ = oracle.decode_workload(w)
    assert np.max(np.abs(out[:, 17] - 1.0)) < 1e-14
    assert np.max(np.abs(out[:, 400] + 2.0)) < 1e-14


def test_empty_sequence():
    w = inputs.make("v3", B=2, H=4, L=[0, 5], seed=9)
    out, lse = oracle.decode_workload(w)
    assert np.all(out[:4] == 0) and np.all(np.isneginf(lse[:4]))
    assert np.all(np.isfinite(lse[4:]))


# ---------------------------------------------------------------- invariants

def test_token_permutation_invariance():
    """Attention is a set operation over cached tokens: shuffling the tokens
    of a sequence changes nothing (up to summation order)."""
    w = inputs.make("v3", B=1, H=8, L=[333], seed=12, q_std=2.0)
    out0, lse0 = oracle.decode_workload(w)
    K = _gather_logical(w, 0).to(torch.bfloat16)
    perm = torch.randperm(333, generator=torch.Generator().manual_seed(1))
    Kp = K[perm]
    cache = torch.zeros_like(w.cache)
    for t in range(333):
        cache[int(w.block_table[0, t // 64]), t % 64] = Kp[t]
    w.cache = cache
    out1, lse1 = oracle.decode_workload(w)
    assert np.max(np.abs(out0 - out1)) < 1e-12
    assert np.max(np.abs(lse0 - lse1)) < 1e-12


@pytest.mark.parametrize("cache", ["bf16", "fp8"])
def test_block_relocation_is_bit_exact(cache):
    """The same logical cache at other physical blocks gives identical bits."""
    w = inputs.make("v3", B=3, H=8, L=[200, 64, 129], cache=cache, seed=13, extra_blocks=5)
    w2 = inputs.relocate(w, seed=99)
    assert not torch.equal(w.block_table, w2.block_table)
    o1, l1 = oracle.decode_workload(w)
    o2, l2 = oracle.decode_workload(w2)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_split_then_combine_equals_unsplit():
    w = inputs.make("v3", B=2, H=4, L=[500, 70], seed=14, q_std=3.0)
    full, lfull = oracle.decode_workload(w)
    cuts = {0: [0, 64, 65, 200, 200, 499, 500], 1: [0, 1, 70]}
    for b, c in cuts.items():
        for h in range(4):
            units = np.array([[b, h, c[i], c[i + 1]] for i in range(len(c) - 1)], np.int32)
            op, lp = oracle.decode_units(q=w.q, cache=w.cache, block_table=w.block_table,
                                         seq_lens=w.seq_lens, num_blocks=w.num_blocks,
                                         softmax_scale=w.softmax_scale, units=units)
            o, l = oracle.combine(op[None], lp[None])
            i = b * 4 + h
            assert np.max(np.abs(o[0] - full[i])) < 1e-12
            assert abs(l[0] - lfull[i]) < 1e-12


def test_combine_edge_cases():
    rng = np.random.default_rng(0)
    o = rng.standard_normal((3, 4, 512))
    lse = rng.standard_normal((3, 4))
    lse[0, :] = -np.inf                      # row 0: nothing at all
    lse[1, 1:] = -np.inf                     # row 1: one live piece
    out, l = oracle.combine(o, lse)
    assert np.all(out[0] == 0) and np.isneginf(l[0])
    assert np.max(np.abs(out[1] - o[1, 0])) < 1e-15 and l[1] == lse[1, 0]
    # row 2: closed form with numpy's logaddexp (library) for the merged lse
    ref_l = np.logaddexp.reduce(lse[2])
    assert abs(l[2] - ref_l) < 1e-13
    ref_o = (np.exp(lse[2] - ref_l)[:, None] * o[2]).sum(0)
    assert np.max(np.abs(out[2] - ref_o)) < 1e-13


def test_fp8_cache_equals_f64_cache_of_dequantised_values():
    """The fp8 oracle reads code * scale[block]; compare with the f64 oracle
    run on values dequantised by torch (library E4M3 conversion)."""
    w = inputs.make("fp8", B=2, H=8, L=[150, 64], seed=15, extra_blocks=1)
    out8, l8 = oracle.decode_workload(w)
    deq = w.cache.view(torch.float8_e4m3fn).double() * w.block_scale.double()[:, None, None]
    f64 = torch.cat([deq, w.k_rope.double()], dim=2).numpy()
    units = oracle.all_units(w.B, w.H)
    o64, l64 = oracle.decode_units(q=w.q, cache=f64, cache_kind="f64", block_table=w.block_table,
                                   seq_lens=w.seq_lens, num_blocks=w.num_blocks,
                                   softmax_scale=w.softmax_scale, units=units)
    assert np.max(np.abs(out8 - o64)) < 1e-15 and np.max(np.abs(l8 - l64)) < 1e-15


def test_bad_block_id_is_reported():
    w = inputs.make("v3", B=1, H=2, L=[100], seed=16)
    w.block_table[0, 1] = w.num_blocks + 3
    with pytest.raises(RuntimeError):
        oracle.decode_workload(w)


def test_absorb_q_matches_library_matmul():
    w = inputs.make("v3", B=3, H=8, L=[1, 1, 1], seed=17)
    ref = torch.einsum("bhd,hdc->bhc", w.q_nope.double(), w.w_uk.double()).numpy()
    got = oracle.absorb_q(w.q_nope, w.w_uk)
    assert np.max(np.abs(got - ref)) < 1e-12


def test_absorb_o_matches_library_matmul():
    """Output absorption (Empirical Gains: W^UV folded into the output
    projection): out[b,h,:] = W_UV[h] . o_latent[b,h,:]."""
    w = inputs.make("v3", B=3, H=8, L=[1, 1, 1], seed=18)
    o = (torch.randn((3, 8, 512), generator=torch.Generator().manual_seed(3)) * 0.05).to(torch.bfloat16)
    ref = torch.einsum("hdc,bhc->bhd", w.w_uv.double(), o.double()).numpy()
    got = oracle.absorb_o(o, w.w_uv)
    assert got.shape == (3, 8, 128)
    assert np.max(np.abs(got - ref)) < 1e-12


def test_absorb_o_one_hot_rows_select_latent_columns():
    """W_UV[h][d] = e_{4d + h % 4} picks one latent column per output: exact."""
    B, H = 2, 4
    w_uv = torch.zeros((H, 128, 512), dtype=torch.bfloat16)
    for h in range(H):
        for d in range(128):
            w_uv[h, d, 4 * d + h % 4] = 1.0
    o = torch.randn((B, H, 512), generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    got = oracle.absorb_o(o, w_uv)
    for h in range(H):
        assert np.array_equal(got[:, h, :], o[:, h, (h % 4)::4].double().numpy())


def test_absorbed_decode_then_output_absorption_equals_naive_heads():
    """Chaining the two absorbed steps on bf16-rounded inputs reproduces the
    naive per-head attention output (the unabsorbed form) to bf16 input
    rounding: the decode in f64 on the cache, then W_UV on its output."""
    H, L = 16, 200
    raw = inputs.raw_tiny_fp32(seed=1, H=H, L=L)
    raw = {k: v.double().numpy() for k, v in raw.items()}
    scale = 1.0 / math.sqrt(192)
    o_naive, _ = naive.naive_mha(raw["c_kv"], raw["k_r"], raw["q_nope"], raw["q_r"],
                                 raw["w_uk"], raw["w_uv"], scale, q_pos=L - 1)
    k_rot = naive.rope(raw["k_r"], np.arange(L))
    rows = np.concatenate([raw["c_kv"], k_rot], axis=1)
    cache, table, NB = _paged_f64(rows, seed=7)
    q_abs = np.einsum("hd,hdc->hc", raw["q_nope"], raw["w_uk"])
    q = np.concatenate([q_abs, naive.rope(raw["q_r"], np.full(H, L - 1))], axis=1)[None]
    o_lat, _ = oracle.decode_units(q=q, q_kind="f64", cache=cache, cache_kind="f64",
                                   block_table=table, seq_lens=np.array([L], np.int32),
                                   num_blocks=NB, softmax_scale=scale, units=oracle.all_units(1, H))
    o_bf = torch.from_numpy(o_lat.reshape(1, H, 512)).to(torch.bfloat16)
    w_uv_bf = torch.from_numpy(raw["w_uv"]).to(torch.bfloat16)
    got = oracle.absorb_o(o_bf, w_uv_bf)[0]
    # bf16 rounding of o_latent and W_UV only: relative error a few 2^-9
    err = np.linalg.norm(got - o_naive) / np.linalg.norm(o_naive)
    assert err < 1e-2
    # and without the rounding the chain is exact
    exact = np.einsum("hdc,hc->hd", raw["w_uv"], o_lat.reshape(H, 512))
    assert np.max(np.abs(exact - o_naive)) < 1e-10


# ---------------------------------------------------------------- page numbers

def test_cache_size_closed_forms_match_page_values():
    g = json.load(open(os.path.join(GOLDEN, "deepseek_v2_cache_sizes.json")))
    d = g["dims"]
    n_h, d_h, d_c, d_r = d["n_h"], d["d_h"], d["d_c"], d["d_h_R"]
    assert d_c == g["dims_as_printed"]["d_c_over_d_h"] * d_h
    assert d_r == g["dims_as_printed"]["d_h_R_over_d_h"] * d_h
    mla = layout.cache_elements_per_token("mla", d_c=d_c, d_h_r=d_r)
    assert mla == layout.D_ROW == 576
    assert mla / d_h == g["mla_elements_per_token_over_d_h"]
    assert layout.equivalent_gqa_groups(d_h=d_h, d_c=d_c, d_h_r=d_r) == g["equivalent_gqa_groups"]
    # the GQA form with 2.25 groups reproduces MLA's footprint exactly
    assert 2 * g["equivalent_gqa_groups"] * d_h == mla
    assert layout.cache_elements_per_token("mha", n_h=n_h, d_h=d_h) == 2 * 128 * 128
    assert layout.cache_elements_per_token("mqa", d_h=d_h) == 256
    assert layout.cache_elements_per_token("mla", layers=60) == 576 * 60
    assert layout.bytes_per_token("bf16") == 1152 and layout.bytes_per_token("fp8") == 640
