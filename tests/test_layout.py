"""The benchmark's algorithmic byte and FLOP counts (mla_latent_kv_25_b200/
layout.py) against the figures of the measurement plan for the workloads:
cache rows of every token once plus the query, output and lse (and one fp32
scale per block for the fp8 cache); FLOPs 2*H*sum(L)*(576 + 512)."""
import pytest

from mla_latent_kv_25_b200 import inputs, layout

# workload: (bytes, flops) as stated by the measurement plan (MB / GFLOP, rounded)
PLAN = {"v3": (319.85e6, 73.01e9), "long": (605.10e6, 146.03e9), "fp8": (689.01e6, 292.06e9)}


@pytest.mark.parametrize("name", sorted(PLAN))
def test_algorithmic_bytes_and_flops_match_the_plan(name):
    cfg = inputs.CONFIGS[name]
    B, H = cfg["B"], cfg["H"]
    tokens = B * cfg["L"]
    blocks = B * ((cfg["L"] + 63) // 64)
    kind = "fp8" if name == "fp8" else "bf16"
    b = layout.decode_algorithmic_bytes(tokens, B, H, kind, num_blocks_read=blocks)
    f = layout.decode_flops(tokens, H)
    want_b, want_f = PLAN[name]
    assert abs(b - want_b) <= 0.005e6, (b, want_b)
    assert abs(f - want_f) <= 0.005e9, (f, want_f)


def test_v3_bytes_exactly():
    # 262,144 rows of 1152 B, query 64*128*1152 B, output and lse 64*128*(1024 + 4) B
    assert layout.decode_algorithmic_bytes(64 * 4096, 64, 128, "bf16") == 319_848_448
