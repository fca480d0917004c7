"""Pins of the cache-writer oracle (oracle/cache.py) against the format
definitions and library routines."""
import numpy as np
import torch

from oracle import cache, naive


def _bf(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_e4m3_round_matches_torch_including_ties():
    rng = np.random.default_rng(0)
    vals = np.sort(cache._VALS)
    mids = (vals[1:] + vals[:-1]) / 2          # exact halfway points: ties
    x = np.concatenate([rng.standard_normal(5000) * 60, mids, -mids, [0.0, -0.0, 500.0, -1e4, 448.0]])
    ref = torch.from_numpy(np.clip(x, -448, 448)).float().to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = cache.e4m3_round(x.astype(np.float32))
    assert np.array_equal(got, ref)


def test_quantize_blocks_scale_extremes_and_error_bound():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, 64, 512)) * np.array([0.02, 3.0, 0.0])[:, None, None]
    x[0, 5, 7] = -0.5                            # the amax element of block 0
    codes, scale = cache.quantize_e4m3_blocks(_bf(x))
    xb = torch.from_numpy(x).float().to(torch.bfloat16).float().numpy()
    assert scale[2] == 1.0 and np.all((codes[2] & 0x7F) == 0)  # all-zero block (signed zeros)
    assert codes[0, 5, 7] == 0xFE                          # -448: the amax maps to the largest code
    dec = np.vectorize(lambda c: float(torch.tensor([c], dtype=torch.uint8).view(torch.float8_e4m3fn).float()))
    for i in (0, 1):
        assert scale[i] == np.float32(np.float32(np.abs(xb[i]).max()) / np.float32(448.0))
        y = dec(codes[i]) * scale[i]
        big = np.abs(xb[i]) > scale[i] * 2.0 ** -6     # normal range: relative error <= 2^-4
        assert np.all(np.abs(y - xb[i])[big] <= np.abs(xb[i])[big] * 2.0 ** -4 + 1e-30)


def test_append_rows_placement_and_rope():
    rng = np.random.default_rng(2)
    T, B = 6, 3
    table = np.array([[4, 1, -1], [0, 2, 3], [5, -1, -1]], np.int32)
    seq = np.array([0, 1, 1, 2, 0, 1])
    pos = np.array([0, 64, 191, 63, 70, 128])
    ck = _bf(rng.standard_normal((T, 512)))
    kr = _bf(rng.standard_normal((T, 64)))
    blocks, rows, data = cache.append(ck, kr, seq, pos, table)
    assert blocks.tolist() == [4, 2, 3, 5, 1, 3]
    assert rows.tolist() == [0, 0, 63, 63, 6, 0]
    ckf = cache._bf16_to_f64(ck)
    krf = cache._bf16_to_f64(kr)
    assert np.array_equal(data[:, :512], ckf)                    # latent copied exactly
    assert np.array_equal(data[0, 512:], krf[0])                 # position 0: no rotation
    n_in = np.hypot(krf[:, 0::2], krf[:, 1::2])
    n_out = np.hypot(data[:, 512::2], data[:, 513::2])
    assert np.max(np.abs(n_in - n_out)) < 1e-12                  # rotations keep pair norms
    # the rotated key scores by relative position only (eeumee.net, RoPE)
    q = rng.standard_normal(64)
    s1 = naive.rope(q, 200) @ naive.rope(krf[1], 64)
    s2 = naive.rope(q, 136) @ naive.rope(krf[1], 0)
    assert abs(s1 - s2) < 1e-10
