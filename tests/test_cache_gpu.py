"""GPU parity of the cache writers (mla_cache_append, mla_cache_quantize_fp8)
through the C ABI against the oracle's cache writers."""
import numpy as np
import pytest
import torch

import oracle
from oracle import cache as cache_oracle
from mla_latent_kv_25_b200 import binding, inputs
from tests._util import assert_close, to_np

pytestmark = pytest.mark.gpu


def _u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _append_case(seed, NB, table, seq, pos):
    g = torch.Generator().manual_seed(seed)
    T = len(seq)
    cache = torch.randn((NB, 64, 576), generator=g).to(torch.bfloat16)
    ck = (torch.randn((T, 512), generator=g) * 0.2).to(torch.bfloat16)
    kr = torch.randn((T, 64), generator=g).to(torch.bfloat16)
    table = torch.tensor(table, dtype=torch.int32)
    seq = torch.tensor(seq, dtype=torch.int32)
    pos = torch.tensor(pos, dtype=torch.int32)
    dev = cache.cuda()
    binding.mla_cache_append(ck.cuda(), kr.cuda(), seq.cuda(), pos.cuda(), table.cuda(), dev)
    err = binding.mla_cache_get_error()
    return cache, ck, kr, table, seq, pos, dev.cpu(), err


def test_cache_append_places_rows_and_rotates_keys():
    table = [[4, 1, 7, -1], [0, 2, 3, 9], [5, 11, -1, -1]]
    seq = [0, 1, 1, 2, 0, 1, 2, 0]
    pos = [0, 64, 191, 63, 70, 255, 127, 190]
    before, ck, kr, table, seq, pos, got, err = _append_case(40, 12, table, seq, pos)
    assert err == 0
    blocks, rows, data = cache_oracle.append(_u16(ck), _u16(kr), seq.numpy(), pos.numpy(), table.numpy())
    touched = torch.zeros((12, 64), dtype=torch.bool)
    for t in range(len(seq)):
        b, r = int(blocks[t]), int(rows[t])
        touched[b, r] = True
        assert torch.equal(got[b, r, :512].view(torch.int16), ck[t].view(torch.int16))  # latent exact
        assert_close(got[b, r, 512:].float().numpy()[None], data[t, 512:][None], f"rope t={t}")
    # every other row is untouched, bit for bit
    assert torch.equal(got[~touched].view(torch.int16), before[~touched].view(torch.int16))


def test_cache_append_long_positions_keep_rope_accuracy():
    mb = 2048
    table = [[-1] * mb]
    table[0][mb - 1] = 3
    table[0][1000] = 1
    before, ck, kr, table, seq, pos, got, err = _append_case(41, 4, table, [0, 0], [131071, 64000 + 5])
    assert err == 0
    blocks, rows, data = cache_oracle.append(_u16(ck), _u16(kr), seq.numpy(), pos.numpy(), table.numpy())
    for t in range(2):
        assert_close(got[int(blocks[t]), int(rows[t]), 512:].float().numpy()[None], data[t, 512:][None],
                     "long-position rope")


def test_cache_append_reports_bad_ids_and_writes_nothing():
    table = [[2, -1], [7, 0]]
    before, _, _, _, _, _, got, err = _append_case(42, 4, table, [0, 1, 0], [64, 10, 200])
    # (0, 64): table entry -1 -> bad block; (1, 10): block 7 >= num_blocks -> bad block;
    # (0, 200): beyond the table -> out of range
    assert err & binding.DEVERR_BAD_BLOCK
    assert err & binding.DEVERR_SEQ_TOO_LONG
    assert torch.equal(got.view(torch.int16), before.view(torch.int16))


def _quantize_case():
    g = torch.Generator().manual_seed(43)
    NB = 8
    cache = torch.randn((NB, 64, 576), generator=g) * 0.05
    cache[2, :, :512] = 0.0                      # an all-zero latent block
    cache[5] *= 2000.0                           # a large-valued block
    cache = cache.to(torch.bfloat16)
    blocks = torch.tensor([5, 0, 2, 7], dtype=torch.int32)
    codes = torch.full((NB, 64, 512), 0xAA, dtype=torch.uint8, device="cuda")
    k_rope = torch.full((NB, 64, 64), 9.0, dtype=torch.bfloat16, device="cuda")
    scale = torch.full((NB,), -1.0, dtype=torch.float32, device="cuda")
    binding.mla_cache_quantize_fp8(cache.cuda(), blocks.cuda(), codes, k_rope, scale)
    err = binding.mla_cache_get_error()
    return NB, cache, blocks, codes.cpu(), k_rope.cpu(), scale.cpu(), err


def test_cache_quantize_fp8_bit_exact():
    """Codes and scales are integers decided in fp32 on both sides: bit-exact."""
    NB, cache, blocks, c, kr, sc, err = _quantize_case()
    assert err == 0
    ref_codes, ref_scale = cache_oracle.quantize_e4m3_blocks(_u16(cache[blocks.long(), :, :512]))
    for i, b in enumerate(blocks.tolist()):
        bad = int((c[b].numpy() != ref_codes[i]).sum())
        assert bad == 0, f"block {b}: {bad} codes differ"
        assert sc[b].item() == float(ref_scale[i]), f"block {b} scale {sc[b].item()} vs {ref_scale[i]}"
        assert torch.equal(kr[b].view(torch.int16), cache[b, :, 512:].view(torch.int16))
    for b in (1, 3, 4, 6):                       # not listed: untouched
        assert torch.all(c[b] == 0xAA) and torch.all(kr[b] == 9.0) and sc[b].item() == -1.0


def test_quantized_blocks_decode_like_any_fp8_cache():
    NB, cache, blocks, c, kr, sc, err = _quantize_case()
    assert err == 0
    w = inputs.make("fp8", B=2, H=16, L=[128, 64], seed=44)
    w.num_blocks = NB
    w.cache, w.k_rope, w.block_scale = c, kr, sc
    w.block_table = torch.tensor([[0, 7], [2, -1]], dtype=torch.int32)  # normally scaled blocks
    d = binding.to_device(w)
    out, lse, ws = binding.decode_device(d, w.softmax_scale, num_splits=2)
    assert binding.mla_get_device_error(ws) == 0
    ro, rl = oracle.decode_workload(w)
    assert_close(to_np(out).reshape(-1, 512), ro, "decode of quantized blocks")
    assert_close(to_np(lse).reshape(-1), rl, "lse of quantized blocks")
