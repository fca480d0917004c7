"""Thin ctypes binding of libmla.so (include/mla.h).

Argument marshalling only: every function checks dtypes, shapes and devices
of torch tensors, passes their device pointers and the current CUDA stream
to the C entry point of the same name, and raises on a non-OK status.  All
arithmetic happens in the CUDA kernels; nothing here computes any part of
the method, and there is no fallback when the library is missing.
"""
from __future__ import annotations

import ctypes
import threading

import torch

from . import build as _build

_lock = threading.Lock()
_lib = None

MLA_OK = 0
STATUS = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED",
          3: "MLA_ERR_WORKSPACE_TOO_SMALL", 4: "MLA_ERR_CUDA", 5: "MLA_ERR_DEVICE"}
MLA_CACHE_BF16 = 0
MLA_CACHE_FP8_E4M3 = 1
DEVERR_BAD_BLOCK = 0x1
DEVERR_SEQ_TOO_LONG = 0x2
DEVERR_TIMEOUT = 0x4
DEVERR_BAD_PIECES = 0x8

# every symbol include/mla.h declares
EXPORTS = ("mla_absorb_q", "mla_absorb_o", "mla_absorb_get_error", "mla_cache_append",
           "mla_cache_quantize_fp8", "mla_cache_get_error", "mla_set_wait_limit", "mla_decode_multi",
           "mla_decode_workspace_bytes", "mla_decode_fp8_workspace_bytes", "mla_decode",
           "mla_combine", "mla_get_device_error", "mla_status_string", "mla_num_sms",
           "mla_decode_noalloc", "mla_decode_noalloc_get_error", "mla_last_error_string")


class MLAError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str = ""):
        msg = f"{fn} returned {STATUS.get(status, status)}"
        super().__init__(msg + (f" ({detail})" if detail else ""))
        self.status = status


def library_path() -> str:
    return _build.LIB


def load():
    """Load libmla.so (building it in-tree with nvcc first if it is absent or
    stale).  Raises if it cannot be built or loaded."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not _build.up_to_date():
            _build.build()
        L = ctypes.CDLL(_build.LIB)
        vp, i32, u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.mla_absorb_q.restype = i32
        L.mla_absorb_q.argtypes = [vp, vp, vp, vp, i32, i32, i32, vp]
        L.mla_absorb_o.restype = i32
        L.mla_absorb_o.argtypes = [vp, vp, vp, i32, i32, i32, vp]
        L.mla_decode_multi.restype = i32
        L.mla_decode_multi.argtypes = [vp, i32, vp, vp, vp, i32, i32, i32, i32, ctypes.c_float, vp, vp,
                                       vp, u64, i32, vp]
        L.mla_set_wait_limit.restype = ctypes.c_longlong
        L.mla_set_wait_limit.argtypes = [ctypes.c_longlong]
        L.mla_cache_append.restype = i32
        L.mla_cache_append.argtypes = [vp, vp, vp, vp, i32, vp, i32, i32, i32, vp, vp]
        L.mla_cache_quantize_fp8.restype = i32
        L.mla_cache_quantize_fp8.argtypes = [vp, vp, i32, i32, vp, vp, vp, vp]
        L.mla_cache_get_error.restype = i32
        L.mla_cache_get_error.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
        L.mla_absorb_get_error.restype = i32
        L.mla_absorb_get_error.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
        L.mla_decode_workspace_bytes.restype = u64
        L.mla_decode_workspace_bytes.argtypes = [i32, i32, i32]
        L.mla_decode_fp8_workspace_bytes.restype = u64
        L.mla_decode_fp8_workspace_bytes.argtypes = [i32, i32, i32, i32]
        L.mla_decode.restype = i32
        L.mla_decode.argtypes = [vp, i32, vp, vp, vp, vp, vp, i32, i32, i32, i32, ctypes.c_float,
                                 vp, vp, vp, u64, i32, vp]
        L.mla_combine.restype = i32
        L.mla_combine.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp]
        L.mla_get_device_error.restype = i32
        L.mla_get_device_error.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32)]
        L.mla_status_string.restype = ctypes.c_char_p
        L.mla_status_string.argtypes = [i32]
        L.mla_num_sms.restype = i32
        L.mla_num_sms.argtypes = []
        L.mla_last_error_string.restype = ctypes.c_char_p
        L.mla_last_error_string.argtypes = []
        L.mla_decode_noalloc.restype = i32
        L.mla_decode_noalloc.argtypes = [vp, i32, vp, vp, vp, vp, vp, i32, i32, i32, i32,
                                         ctypes.c_float, vp, vp, i32, vp]
        L.mla_decode_noalloc_get_error.restype = i32
        L.mla_decode_noalloc_get_error.argtypes = [vp, vp]
        _lib = L
        return L


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn, status):
    if status != MLA_OK:
        detail = load().mla_last_error_string().decode() if status == 4 else ""
        raise MLAError(fn, status, detail)


def _need(t, name, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")


def mla_status_string(status: int) -> str:
    return load().mla_status_string(int(status)).decode()


def mla_num_sms() -> int:
    return int(load().mla_num_sms())


def mla_decode_workspace_bytes(B: int, H: int, num_splits: int = 0) -> int:
    return int(load().mla_decode_workspace_bytes(int(B), int(H), int(num_splits)))


def mla_decode_fp8_workspace_bytes(B: int, H: int, max_blocks: int, num_splits: int = 0) -> int:
    return int(load().mla_decode_fp8_workspace_bytes(int(B), int(H), int(max_blocks),
                                                     int(num_splits)))


def alloc_workspace(B: int, H: int, num_splits: int = 0, device=None,
                    fp8_max_blocks: int | None = None) -> torch.Tensor:
    """Zero-filled device workspace of the size mla_decode needs.  With
    ``fp8_max_blocks`` (the block table's width) it also holds the widened
    bf16 copy that runs an fp8 cache on the tensor cores."""
    if fp8_max_blocks is None:
        n = mla_decode_workspace_bytes(B, H, num_splits)
        fn = "mla_decode_workspace_bytes"
    else:
        n = mla_decode_fp8_workspace_bytes(B, H, fp8_max_blocks, num_splits)
        fn = "mla_decode_fp8_workspace_bytes"
    if n == 0:
        raise MLAError(fn, 1)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def mla_absorb_q(q_nope, w_uk, q_rope, q_out, stream=None):
    """q_out[b,h,:512] = q_nope[b,h] . w_uk[h]; q_out[b,h,512:576] = q_rope[b,h]."""
    B, H = int(q_nope.shape[0]), int(q_nope.shape[1])
    _need(q_nope, "q_nope", torch.bfloat16, (B, H, 128))
    _need(w_uk, "w_uk", torch.bfloat16, (H, 128, 512))
    if q_rope is not None:
        _need(q_rope, "q_rope", torch.bfloat16, (B, H, 64))
    _need(q_out, "q_out", torch.bfloat16)
    if q_out.dim() != 3 or tuple(q_out.shape[:2]) != (B, H):
        raise ValueError("q_out must be [B,H,ldq]")
    ldq = int(q_out.shape[2])
    _check("mla_absorb_q", load().mla_absorb_q(_ptr(q_nope), _ptr(w_uk), _ptr(q_rope), _ptr(q_out),
                                               ldq, B, H, _stream(stream)))
    return q_out


def mla_absorb_o(o_latent, w_uv, out, stream=None):
    """out[b,h,:] = w_uv[h] . o_latent[b,h,:] (the output absorption)."""
    B, H = int(o_latent.shape[0]), int(o_latent.shape[1])
    _need(o_latent, "o_latent", torch.bfloat16, (B, H, 512))
    _need(w_uv, "w_uv", torch.bfloat16, (H, 128, 512))
    _need(out, "out", torch.bfloat16)
    if out.dim() != 3 or tuple(out.shape[:2]) != (B, H):
        raise ValueError("out must be [B,H,ldo]")
    _check("mla_absorb_o", load().mla_absorb_o(_ptr(o_latent), _ptr(w_uv), _ptr(out),
                                               int(out.shape[2]), B, H, _stream(stream)))
    return out


def mla_cache_append(c_kv, k_r, seq_idx, pos, block_table, cache, stream=None):
    """Write [c_kv | RoPE(k_r, pos)] rows of new tokens into the paged bf16 cache."""
    T = int(c_kv.shape[0])
    _need(c_kv, "c_kv", torch.bfloat16, (T, 512))
    _need(k_r, "k_r", torch.bfloat16, (T, 64))
    _need(seq_idx, "seq_idx", torch.int32, (T,))
    _need(pos, "pos", torch.int32, (T,))
    _need(block_table, "block_table", torch.int32)
    _need(cache, "cache", torch.bfloat16)
    B, mb = int(block_table.shape[0]), int(block_table.shape[1])
    _check("mla_cache_append", load().mla_cache_append(
        _ptr(c_kv), _ptr(k_r), _ptr(seq_idx), _ptr(pos), T, _ptr(block_table), B, mb,
        int(cache.shape[0]), _ptr(cache), _stream(stream)))
    return cache


def mla_cache_quantize_fp8(cache_bf16, blocks, codes, k_rope, block_scale, stream=None):
    """Convert the listed blocks of a bf16 cache to the fp8 layout."""
    _need(cache_bf16, "cache_bf16", torch.bfloat16)
    _need(blocks, "blocks", torch.int32)
    _need(codes, "codes", torch.uint8)
    _need(k_rope, "k_rope", torch.bfloat16)
    _need(block_scale, "block_scale", torch.float32)
    _check("mla_cache_quantize_fp8", load().mla_cache_quantize_fp8(
        _ptr(cache_bf16), _ptr(blocks), int(blocks.numel()), int(cache_bf16.shape[0]), _ptr(codes),
        _ptr(k_rope), _ptr(block_scale), _stream(stream)))
    return codes, k_rope, block_scale


def mla_decode_multi(q, cache, block_table, seq_lens, softmax_scale, out, lse, workspace, *,
                     num_splits=0, stream=None):
    """Decode q_len query tokens per sequence (q [B,q_len,H,576], bf16 cache)."""
    B, q_len, H = int(q.shape[0]), int(q.shape[1]), int(q.shape[2])
    _need(q, "q", torch.bfloat16, (B, q_len, H, 576))
    _need(cache, "cache", torch.bfloat16)
    _need(block_table, "block_table", torch.int32)
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    _need(out, "out", torch.bfloat16, (B, q_len, H, 512))
    _need(lse, "lse", torch.float32, (B, q_len, H))
    _need(workspace, "workspace", torch.uint8)
    _check("mla_decode_multi", load().mla_decode_multi(
        _ptr(q), q_len, _ptr(cache), _ptr(block_table), _ptr(seq_lens), B, H, int(cache.shape[0]),
        int(block_table.shape[1]), float(softmax_scale), _ptr(out), _ptr(lse), _ptr(workspace),
        int(workspace.numel()), int(num_splits), _stream(stream)))
    return out, lse


def mla_set_wait_limit(cycles: int) -> int:
    """Bound of the decode kernels' waits in SM cycles (<= 0: the default);
    returns the previous bound."""
    return int(load().mla_set_wait_limit(int(cycles)))


def mla_cache_get_error(stream=None) -> int:
    """Synchronise the stream, return and clear the cache writers' error bits."""
    v = ctypes.c_uint32(0)
    _check("mla_cache_get_error", load().mla_cache_get_error(_stream(stream), ctypes.byref(v)))
    return int(v.value)


def mla_absorb_get_error(stream=None) -> int:
    """Synchronise the stream, return and clear the absorption kernel's error bits."""
    v = ctypes.c_uint32(0)
    _check("mla_absorb_get_error", load().mla_absorb_get_error(_stream(stream), ctypes.byref(v)))
    return int(v.value)


def mla_decode(q, cache, block_table, seq_lens, softmax_scale, out, lse, workspace, *,
               k_rope=None, block_scale=None, num_splits=0, stream=None):
    """Decode attention over the paged latent cache (see include/mla.h)."""
    B, H = int(q.shape[0]), int(q.shape[1])
    _need(q, "q", torch.bfloat16, (B, H, 576))
    if cache.dtype == torch.bfloat16:
        kind = MLA_CACHE_BF16
        _need(cache, "cache", torch.bfloat16)
        if cache.dim() != 3 or tuple(cache.shape[1:]) != (64, 576):
            raise ValueError("bf16 cache must be [num_blocks,64,576]")
    elif cache.dtype == torch.uint8:
        kind = MLA_CACHE_FP8_E4M3
        _need(cache, "cache", torch.uint8)
        if cache.dim() != 3 or tuple(cache.shape[1:]) != (64, 512):
            raise ValueError("fp8 cache must be [num_blocks,64,512] uint8")
        NB = int(cache.shape[0])
        _need(k_rope, "k_rope", torch.bfloat16, (NB, 64, 64))
        _need(block_scale, "block_scale", torch.float32, (NB,))
    else:
        raise TypeError("cache must be bf16 or uint8 (E4M3 codes)")
    NB = int(cache.shape[0])
    _need(block_table, "block_table", torch.int32)
    if block_table.dim() != 2 or int(block_table.shape[0]) != B:
        raise ValueError("block_table must be [B,max_blocks]")
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    _need(out, "out", torch.bfloat16, (B, H, 512))
    _need(lse, "lse", torch.float32, (B, H))
    _need(workspace, "workspace", torch.uint8)
    st = load().mla_decode(_ptr(q), kind, _ptr(cache), _ptr(k_rope), _ptr(block_scale),
                           _ptr(block_table), _ptr(seq_lens), B, H, NB, int(block_table.shape[1]),
                           float(softmax_scale), _ptr(out), _ptr(lse), _ptr(workspace),
                           int(workspace.numel()), int(num_splits), _stream(stream))
    _check("mla_decode", st)
    return out, lse


def mla_decode_noalloc(q, cache, block_table, seq_lens, softmax_scale, out, lse, *,
                       k_rope=None, block_scale=None, num_splits=0, stream=None):
    """mla_decode with the library's built-in scratch instead of a caller
    workspace, for callers that cannot allocate device memory (see
    include/mla.h): only inputs and outputs are passed."""
    B, H = int(q.shape[0]), int(q.shape[1])
    _need(q, "q", torch.bfloat16, (B, H, 576))
    kind = MLA_CACHE_BF16 if cache.dtype == torch.bfloat16 else MLA_CACHE_FP8_E4M3
    _need(cache, "cache", cache.dtype)
    _need(block_table, "block_table", torch.int32)
    _need(seq_lens, "seq_lens", torch.int32, (B,))
    _need(out, "out", torch.bfloat16, (B, H, 512))
    _need(lse, "lse", torch.float32, (B, H))
    st = load().mla_decode_noalloc(_ptr(q), kind, _ptr(cache), _ptr(k_rope), _ptr(block_scale),
                                   _ptr(block_table), _ptr(seq_lens), B, H, int(cache.shape[0]),
                                   int(block_table.shape[1]), float(softmax_scale), _ptr(out),
                                   _ptr(lse), int(num_splits), _stream(stream))
    _check("mla_decode_noalloc", st)
    return out, lse


def mla_combine(o_part, lse_part, out, lse, stream=None):
    """LSE merge: o_part [B,H,S,512] f32, lse_part [B,H,S] f32 -> out bf16, lse f32."""
    B, H, S = int(lse_part.shape[0]), int(lse_part.shape[1]), int(lse_part.shape[2])
    _need(o_part, "o_part", torch.float32, (B, H, S, 512))
    _need(lse_part, "lse_part", torch.float32, (B, H, S))
    _need(out, "out", torch.bfloat16, (B, H, 512))
    _need(lse, "lse", torch.float32, (B, H))
    _check("mla_combine", load().mla_combine(_ptr(o_part), _ptr(lse_part), B, H, S, _ptr(out),
                                             _ptr(lse), _stream(stream)))
    return out, lse


def mla_decode_noalloc_get_error(stream=None) -> int:
    """Synchronise the stream, return and clear the error bits of the
    built-in scratch of mla_decode_noalloc (current device)."""
    v = ctypes.c_uint32(0)
    _check("mla_decode_noalloc_get_error",
           load().mla_decode_noalloc_get_error(_stream(stream), ctypes.byref(v)))
    return int(v.value)


def mla_get_device_error(workspace, stream=None) -> int:
    """Synchronise the stream, return and clear the device error bits."""
    v = ctypes.c_uint32(0)
    _check("mla_get_device_error",
           load().mla_get_device_error(_ptr(workspace), _stream(stream), ctypes.byref(v)))
    return int(v.value)


# ----------------------------------------------------------------------------
# Convenience: run a Workload from the input generator (tensors moved to GPU).

def to_device(w, device="cuda"):
    """Copy a generated Workload's tensors to the device (returns a dict)."""
    d = dict(q=w.q.to(device), cache=w.cache.to(device), block_table=w.block_table.to(device),
             seq_lens=w.seq_lens.to(device))
    d["k_rope"] = w.k_rope.to(device) if w.k_rope is not None else None
    d["block_scale"] = w.block_scale.to(device) if w.block_scale is not None else None
    if w.q_nope is not None:
        d["q_nope"] = w.q_nope.to(device)
        d["w_uk"] = w.w_uk.to(device)
    if w.w_uv is not None:
        d["w_uv"] = w.w_uv.to(device)
    return d


def decode_device(d, softmax_scale, num_splits=0, workspace=None, stream=None):
    """mla_decode on device tensors from ``to_device``; allocates outputs and,
    unless one is given, the workspace (for an fp8 cache, with room for the
    widened copy, so that it runs on the tensor cores)."""
    B, H = int(d["q"].shape[0]), int(d["q"].shape[1])
    dev = d["q"].device
    out = torch.empty((B, H, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    if workspace is None:
        fp8 = d["cache"].dtype == torch.uint8
        workspace = alloc_workspace(B, H, num_splits, device=dev,
                                    fp8_max_blocks=int(d["block_table"].shape[1]) if fp8 else None)
    mla_decode(d["q"], d["cache"], d["block_table"], d["seq_lens"], softmax_scale, out, lse,
               workspace, k_rope=d["k_rope"], block_scale=d["block_scale"],
               num_splits=num_splits, stream=stream)
    return out, lse, workspace
