"""FP64 CPU oracle for the absorbed MLA decode step.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` are the only callers.  Nothing here is shared
with, or called by, the CUDA path.

Parts:
  * ``mla_oracle.c`` (compiled to ``_build/liboracle.so``): the plain
    definition of absorbed decode attention over the paged latent cache, the
    log-sum-exp merge of split pieces, the query and output absorptions, and the bf16 /
    OCP E4M3 decoders.
  * ``naive.py``: the unabsorbed form (per-head keys and values formed from
    the latent with W_UK / W_UV, RoPE on the decoupled part only, plain
    softmax attention), used to pin the absorbed form.

Every function is pinned by a ``-m "not gpu"`` test against something other
than itself (see tests/test_oracle_pins.py).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mla_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "liboracle.so")
# a prebuilt oracle library to load instead (the mutation test points the pins
# at deliberately broken copies this way); it is used as it is, never rebuilt
_LIB_OVERRIDE = os.environ.get("MLA_ORACLE_LIB")
_lock = threading.Lock()
_lib = None

F64, BF16, E4M3 = 0, 1, 2
D_C, D_R, D_ROW, BLOCK = 512, 64, 576, 64


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (OpenMP, -O2, strict IEEE: no fast-math)."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
               "-o", tmp, _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            if _LIB_OVERRIDE:
                L = ctypes.CDLL(_LIB_OVERRIDE)
            else:
                build()
                L = ctypes.CDLL(_LIB_PATH)
            vp, i32p = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32)
            L.orc_decode_units.restype = ctypes.c_int
            L.orc_decode_units.argtypes = [ctypes.c_int, vp, ctypes.c_int, vp, vp, vp, vp, vp,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_double, vp, ctypes.c_int, vp, vp, ctypes.c_int]
            L.orc_combine.restype = None
            L.orc_combine.argtypes = [vp, vp, ctypes.c_int, ctypes.c_int, vp, vp]
            L.orc_absorb_q.restype = None
            L.orc_absorb_q.argtypes = [vp, vp, ctypes.c_int, ctypes.c_int, vp]
            L.orc_absorb_o.restype = None
            L.orc_absorb_o.argtypes = [vp, vp, ctypes.c_int, ctypes.c_int, vp]
            L.orc_bf16_to_f64.restype = ctypes.c_double
            L.orc_bf16_to_f64.argtypes = [ctypes.c_uint16]
            L.orc_e4m3_to_f64.restype = ctypes.c_double
            L.orc_e4m3_to_f64.argtypes = [ctypes.c_uint8]
            L.orc_max_threads.restype = ctypes.c_int
            _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _np(t, dtype):
    """torch tensor or numpy array -> contiguous numpy array of ``dtype``.
    bf16 tensors are passed as their raw uint16 bit patterns."""
    import torch
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            t = t.view(torch.int16)
        a = t.numpy()
    else:
        a = np.asarray(t)
    a = np.ascontiguousarray(a)
    dt = np.dtype(dtype)
    if a.dtype.kind in "iu" and dt.kind in "iu" and a.dtype.itemsize == dt.itemsize:
        return a.view(dt)
    return np.ascontiguousarray(a.astype(dt))


def bf16_to_f64(bits: int) -> float:
    return lib().orc_bf16_to_f64(int(bits) & 0xFFFF)


def e4m3_to_f64(code: int) -> float:
    return lib().orc_e4m3_to_f64(int(code) & 0xFF)


def max_threads() -> int:
    return int(lib().orc_max_threads())


def decode_units(*, q, cache, block_table, seq_lens, num_blocks, softmax_scale, units,
                 cache_kind="bf16", k_rope=None, block_scale=None, q_kind="bf16",
                 nthreads=0):
    """Run the oracle on ``units`` = int32 [n,4] rows (b, h, t0, t1); t1 = -1
    means the whole sequence.  Returns (out [n,512] f64, lse [n] f64)."""
    L = lib()
    if q_kind == "f64":
        qa, qk = np.ascontiguousarray(q, dtype=np.float64), F64
    else:
        qa, qk = _np(q, np.uint16), BF16
    B, H = int(qa.shape[0]), int(qa.shape[1])
    if cache_kind == "f64":
        ca, ck = np.ascontiguousarray(cache, dtype=np.float64), F64
        kr = sc = None
    elif cache_kind == "bf16":
        ca, ck = _np(cache, np.uint16), BF16
        kr = sc = None
    elif cache_kind == "fp8":
        ca, ck = _np(cache, np.uint8), E4M3
        kr = _np(k_rope, np.uint16)
        sc = _np(block_scale, np.float32)
    else:
        raise ValueError(cache_kind)
    bt = _np(block_table, np.int32)
    sl = _np(seq_lens, np.int32)
    u = np.ascontiguousarray(units, dtype=np.int32).reshape(-1, 4)
    n = int(u.shape[0])
    out = np.zeros((n, D_C), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    rc = L.orc_decode_units(qk, _ptr(qa), ck, _ptr(ca),
                            _ptr(kr) if kr is not None else None,
                            _ptr(sc) if sc is not None else None,
                            _ptr(bt), _ptr(sl), B, H, int(num_blocks), int(bt.shape[1]),
                            float(softmax_scale), _ptr(u), n, _ptr(out), _ptr(lse), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle decode failed with code {rc}")
    return out, lse


def all_units(B: int, H: int) -> np.ndarray:
    b, h = np.meshgrid(np.arange(B), np.arange(H), indexing="ij")
    u = np.stack([b.ravel(), h.ravel(), np.zeros(B * H, int), -np.ones(B * H, int)], axis=1)
    return u.astype(np.int32)


def decode_workload(w, rows=None, nthreads=0):
    """Oracle over a Workload (from the shared input generator).  ``rows`` is
    an optional int array [n,2] of (b, h) pairs; default all B*H rows.
    Returns (out [n,512], lse [n])."""
    if rows is None:
        units = all_units(w.B, w.H)
    else:
        rows = np.asarray(rows, dtype=np.int32).reshape(-1, 2)
        units = np.concatenate([rows, np.zeros((len(rows), 1), np.int32),
                                -np.ones((len(rows), 1), np.int32)], axis=1)
    return decode_units(q=w.q, cache=w.cache, block_table=w.block_table, seq_lens=w.seq_lens,
                        num_blocks=w.num_blocks, softmax_scale=w.softmax_scale, units=units,
                        cache_kind=w.cache_dtype, k_rope=w.k_rope, block_scale=w.block_scale,
                        nthreads=nthreads)


def combine(o_part, lse_part):
    """Log-sum-exp merge: o_part [R,S,512], lse_part [R,S] -> (out [R,512], lse [R])."""
    op = np.ascontiguousarray(o_part, dtype=np.float64)
    lp = np.ascontiguousarray(lse_part, dtype=np.float64)
    R, S = int(lp.shape[0]), int(lp.shape[1])
    out = np.zeros((R, D_C), dtype=np.float64)
    lse = np.zeros((R,), dtype=np.float64)
    lib().orc_combine(_ptr(op), _ptr(lp), R, S, _ptr(out), _ptr(lse))
    return out, lse


def absorb_o(o_latent, w_uv):
    """out[b,h,d] = sum_c W_UV[h,d,c] * o_latent[b,h,c] in double; bf16 inputs."""
    ol = _np(o_latent, np.uint16)
    wv = _np(w_uv, np.uint16)
    B, H = int(ol.shape[0]), int(ol.shape[1])
    out = np.zeros((B, H, 128), dtype=np.float64)
    lib().orc_absorb_o(_ptr(ol), _ptr(wv), B, H, _ptr(out))
    return out


def absorb_q(q_nope, w_uk):
    """q_abs[b,h,:] = q_nope[b,h,:] . W_UK[h] in double; bf16 inputs."""
    qn = _np(q_nope, np.uint16)
    wu = _np(w_uk, np.uint16)
    B, H = int(qn.shape[0]), int(qn.shape[1])
    out = np.zeros((B, H, D_C), dtype=np.float64)
    lib().orc_absorb_q(_ptr(qn), _ptr(wu), B, H, _ptr(out))
    return out
