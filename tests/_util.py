"""Comparison helpers shared by the GPU parity tests."""
import numpy as np
import torch

# Floating-point bar for bf16 outputs: max-abs 2e-2 and relative L2 5e-3
# against the FP64 oracle on the same inputs.
MAX_ABS = 2e-2
REL_L2 = 5e-3


def rel_l2(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def assert_close(got, ref, what="", max_abs=MAX_ABS, rel=REL_L2):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin), f"{what}: finiteness differs"
    if not fin.any():
        return
    d = np.max(np.abs(got[fin] - ref[fin]))
    r = rel_l2(got[fin], ref[fin])
    assert d <= max_abs, f"{what}: max-abs {d:.3e} > {max_abs}"
    assert r <= rel, f"{what}: rel-L2 {r:.3e} > {rel}"


def to_np(t):
    return t.detach().float().cpu().numpy() if t.dtype != torch.float64 else t.cpu().numpy()
