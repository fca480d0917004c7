"""The C-ABI library loads on a machine without a GPU, exports every entry
point include/mla.h declares, and rejects invalid arguments on the host
before touching the device."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

from mla_latent_kv_25_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "mla.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("mla_absorb_q", "mla_decode", "mla_combine", "mla_decode_workspace_bytes",
              "mla_get_device_error", "mla_status_string"):
        assert n in names
    assert set(names) == set(binding.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = binding.load()
    for n in declared_functions():
        assert hasattr(lib, n), n
        assert isinstance(getattr(lib, n), ctypes._CFuncPtr)


def test_error_codes_agree_across_header_kernels_and_binding():
    """The status enum and device error bits of include/mla.h, the kernels'
    error constants (csrc/common.cuh) and the binding's constants agree."""
    hdr = open(os.path.join(ROOT, "include", "mla.h")).read()
    enum = {n: int(v) for n, v in re.findall(r"\b(MLA_(?:OK|ERR_[A-Z_]+))\s*=\s*(\d+)", hdr)}
    assert {binding.STATUS[v]: v for v in binding.STATUS} == enum
    bits = {n: int(v, 16) for n, v in re.findall(r"#define (MLA_DEVERR_[A-Z_]+)\s+0x([0-9a-fA-F]+)u", hdr)}
    assert bits == {"MLA_DEVERR_BAD_BLOCK": binding.DEVERR_BAD_BLOCK,
                    "MLA_DEVERR_SEQ_TOO_LONG": binding.DEVERR_SEQ_TOO_LONG,
                    "MLA_DEVERR_TIMEOUT": binding.DEVERR_TIMEOUT,
                    "MLA_DEVERR_BAD_PIECES": binding.DEVERR_BAD_PIECES}
    common = open(os.path.join(ROOT, "mla_latent_kv_25_b200", "csrc", "common.cuh")).read()
    kern = {n: int(v, 16) for n, v in re.findall(r"constexpr uint32_t (kErr[A-Za-z]+) = 0x([0-9a-fA-F]+)u;", common)}
    assert kern == {"kErrBadBlock": bits["MLA_DEVERR_BAD_BLOCK"], "kErrSeqTooLong": bits["MLA_DEVERR_SEQ_TOO_LONG"],
                    "kErrTimeout": bits["MLA_DEVERR_TIMEOUT"], "kErrBadPieces": bits["MLA_DEVERR_BAD_PIECES"]}


def test_status_strings():
    for code, name in binding.STATUS.items():
        assert binding.mla_status_string(code) == name


def test_workspace_size_and_validation_without_device():
    lib = binding.load()
    # explicit split count: no device query needed
    n1 = lib.mla_decode_workspace_bytes(64, 128, 74)
    n2 = lib.mla_decode_workspace_bytes(64, 128, 148)
    assert n1 > 0 and n2 > n1 and n1 % 256 == 0
    # room for 2 fp32 pieces (512 + lse) per engine and head
    assert n1 >= 2 * 74 * 128 * 513 * 4
    assert lib.mla_decode_workspace_bytes(64, 100, 74) == 0     # H not a multiple of 16
    # multi-token rows above 128 run in 128-row tiles: the workspace of one tile
    assert lib.mla_decode_workspace_bytes(64, 256, 74) == n1
    assert lib.mla_decode_workspace_bytes(64, 1024, 74) == n1
    assert lib.mla_decode_workspace_bytes(64, 192, 74) == 0     # not whole 128-row tiles
    assert lib.mla_decode_workspace_bytes(64, 1152, 74) == 0    # more than 8 tiles
    assert lib.mla_decode_fp8_workspace_bytes(64, 256, 4, 74) == 0  # fp8: one token per sequence
    assert lib.mla_decode_workspace_bytes(0, 128, 74) == 0
    assert lib.mla_decode_workspace_bytes(1, 128, -1) == 0


def _workspace_in_child(env_value):
    code = ("from mla_latent_kv_25_b200 import binding; "
            "print(binding.load().mla_decode_workspace_bytes(64, 128, 0))")
    env = dict(os.environ)
    env.pop("MLA_SPLITS", None)
    if env_value is not None:
        env["MLA_SPLITS"] = env_value
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0, r.stderr[-2000:]
    return int(r.stdout.strip().splitlines()[-1])


def test_env_split_count_replaces_the_automatic_one():
    """MLA_SPLITS=<1..4096> sets the split count that num_splits = 0 means;
    other values leave the automatic count."""
    lib = binding.load()
    auto = _workspace_in_child(None)
    assert _workspace_in_child("5") == lib.mla_decode_workspace_bytes(64, 128, 5)
    assert _workspace_in_child("4096") == lib.mla_decode_workspace_bytes(64, 128, 4096)
    for bad in ("0", "-3", "4097", "abc", "7x", ""):
        assert _workspace_in_child(bad) == auto, bad


def test_fp8_workspace_adds_the_widened_copy():
    """The tensor-core route of the fp8 cache needs the split-KV workspace,
    then a scratch block table (int32 per table entry) and one bf16 block of
    64 x 576 per table entry, each region 256-byte aligned."""
    lib = binding.load()
    for B, H, mb, P in [(64, 128, 256, 74), (3, 32, 5, 3), (1, 16, 1, 1)]:
        base = lib.mla_decode_workspace_bytes(B, H, P)
        table = -(-base // 256) * 256
        cache = -(-(table + 4 * B * mb) // 256) * 256
        assert lib.mla_decode_fp8_workspace_bytes(B, H, mb, P) == cache + B * mb * 64 * 576 * 2
    assert lib.mla_decode_fp8_workspace_bytes(64, 128, 0, 74) == 0        # no table
    assert lib.mla_decode_fp8_workspace_bytes(64, 100, 4, 74) == 0        # bad H
    assert lib.mla_decode_fp8_workspace_bytes(4096, 128, 8192, 74) == 0   # 2^25 blocks > 2^24


@pytest.mark.parametrize("case", ["null_q", "bad_heads", "bad_batch", "fp8_missing_rope",
                                  "bf16_with_scale", "bad_scale", "misaligned"])
def test_decode_rejects_invalid_arguments_on_host(case):
    lib = binding.load()
    P = ctypes.c_void_p
    good = P(4096)
    args = dict(q=good, kind=0, cache=good, k_rope=None, scale=None, table=good, lens=good,
                B=4, H=128, NB=10, maxb=4, sm=0.07, out=good, lse=good, ws=P(256 * 64),
                wsb=1 << 30, splits=2, stream=None)
    if case == "null_q":
        args["q"] = None
    elif case == "bad_heads":
        args["H"] = 40
    elif case == "bad_batch":
        args["B"] = 0
    elif case == "fp8_missing_rope":
        args["kind"] = 1
        args["scale"] = good
    elif case == "bf16_with_scale":
        args["scale"] = good
    elif case == "bad_scale":
        args["sm"] = float("nan")
    elif case == "misaligned":
        args["cache"] = P(4096 + 2)
    st = lib.mla_decode(args["q"], args["kind"], args["cache"], args["k_rope"], args["scale"],
                        args["table"], args["lens"], args["B"], args["H"], args["NB"], args["maxb"],
                        args["sm"], args["out"], args["lse"], args["ws"], args["wsb"],
                        args["splits"], args["stream"])
    assert st == 1, binding.STATUS.get(st, st)


def test_absorb_and_combine_reject_invalid_arguments_on_host():
    lib = binding.load()
    P = ctypes.c_void_p
    g = P(4096)
    assert lib.mla_absorb_q(None, g, None, g, 576, 1, 16, None) == 1
    assert lib.mla_absorb_q(g, g, g, g, 512, 1, 16, None) == 1      # ldq too small for q_rope
    assert lib.mla_absorb_q(g, g, None, g, 516, 1, 16, None) == 1   # ldq not a multiple of 8
    assert lib.mla_absorb_o(None, g, g, 128, 1, 16, None) == 1
    assert lib.mla_absorb_o(g, g, g, 120, 1, 16, None) == 1       # ldo below 128
    assert lib.mla_absorb_o(g, g, g, 132, 1, 16, None) == 1       # ldo not a multiple of 8
    assert lib.mla_absorb_o(g, g, g, 128, 1, 24, None) == 1       # H not a multiple of 16
    assert lib.mla_absorb_o(g, g, P(4100), 128, 1, 16, None) == 1  # misaligned output
    assert lib.mla_absorb_get_error(None, None) == 1
    assert lib.mla_cache_append(None, g, g, g, 1, g, 1, 1, 1, g, None) == 1
    assert lib.mla_cache_append(g, g, g, g, -1, g, 1, 1, 1, g, None) == 1   # negative T
    assert lib.mla_cache_append(P(4100), g, g, g, 1, g, 1, 1, 1, g, None) == 1  # misaligned rows
    assert lib.mla_cache_append(g, g, g, g, 0, g, 1, 1, 1, g, None) == 0    # T = 0: nothing to do
    assert lib.mla_cache_quantize_fp8(None, g, 1, 1, g, g, g, None) == 1
    assert lib.mla_cache_quantize_fp8(g, g, -1, 1, g, g, g, None) == 1      # negative n
    assert lib.mla_cache_quantize_fp8(g, g, 1, 0, g, g, g, None) == 1       # no blocks
    assert lib.mla_cache_get_error(None, None) == 1
    # multi-token decode: q_len * H must be a multiple of 16 and at most 128
    assert lib.mla_decode_multi(g, 0, g, g, g, 1, 16, 1, 1, 0.1, g, g, g, 1 << 20, 0, None) == 1
    assert lib.mla_decode_multi(g, 3, g, g, g, 1, 8, 1, 1, 0.1, g, g, g, 1 << 20, 0, None) == 1
    assert lib.mla_decode_multi(g, 2, g, g, g, 1, 96, 1, 1, 0.1, g, g, g, 1 << 20, 0, None) == 1  # 192 rows: not whole 128-row tiles
    assert lib.mla_decode_multi(g, 3, g, g, g, 1, 128, 1, 1, 0.1, g, g, g, 1 << 20, 9, None) == 3  # tiles need one 128-row workspace
    assert lib.mla_decode_multi(None, 2, g, g, g, 1, 16, 1, 1, 0.1, g, g, g, 1 << 20, 0, None) == 1
    assert lib.mla_combine(None, g, 1, 16, 2, g, g, None) == 1
    assert lib.mla_combine(g, g, 1, 16, 0, g, g, None) == 1
