"""Benchmark of the absorbed MLA decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload v3] [--num-splits P]

One step = one pass of the whole hot path over one batch: mla_absorb_q
(q_nope . W_UK, packed with q_rope) then mla_decode (split-KV decode over the
paged latent cache, then the LSE merge of cut sequences).  Inputs are seeded
synthetic tensors of the DeepSeek-V3 decode shape (B=64, H=128, L=4096, bf16
paged cache in 64-token blocks under a random block permutation), resident in
HBM before timing.  The cache (302 MB) is larger than L2 (126 MB), so no L2
flush is needed between steps.

value = algorithmic bytes of one step (cache rows of every token once, the
query, the output and lse, W_UK and the absorption inputs/outputs) divided by
the device time per step (CUDA events, max over ranks), in GB/s.

Multi-GPU: the decode of independent batches does not exchange anything, so
N ranks run N independent replicas (weak scaling); the only collective is
the max-over-ranks of the timings.

--impl reference times the FP64 CPU oracle on a bounded sample of the same
workload (the reference arm of this method is the oracle).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from mla_latent_kv_25_b200 import inputs, layout  # noqa: E402

METRIC = "MLA decode: cache GB/s and TFLOP/s vs roofline at DeepSeek-V3 shapes, 1 B200"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="v3", choices=list(inputs.CONFIGS))
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra-workloads", action="store_true",
                    help="skip the decode timings of the ragged, long and fp8 configurations")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle sample")
    ap.add_argument("--json-out", default=None,
                    help="also append the result line to this file (rank 0)")
    return ap.parse_args()


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_seed(workload: str, rank: int) -> int:
    """Each replica decodes its own batch: the workload's seed offset by rank."""
    return inputs.CONFIGS[workload]["seed"] + 1000 * rank


def max_over_ranks(values, device):
    """Elementwise max over all ranks of the process group (a no-op for one
    process); every rank gets the result.  Timings are reported as the slowest
    rank's."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_rate(bytes_per_rank_step: float, world: int, step_ms: float) -> float:
    """Whole-job GB/s: the bytes every rank processed per step over the
    (max-over-ranks) step time."""
    return bytes_per_rank_step * world / (step_ms * 1e-3) / 1e9


def absorb_o_line(B: int, H: int, ms: float, hbm_gbs: float) -> dict:
    """Output absorption timed separately: algorithmic bytes = o_latent + W_UV
    + out (bf16)."""
    nbytes = B * H * 512 * 2 + H * 128 * 512 * 2 + B * H * 128 * 2
    achieved = nbytes / (ms * 1e-3) / 1e9
    return {"us_per_launch": round(ms * 1e3, 2), "algorithmic_bytes": nbytes,
            "achieved_gbs": round(achieved, 1), "bound": "hbm",
            "frac": round(achieved / hbm_gbs, 4)}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


DECODE_KERNEL_SOURCES = ("decode_sm100.cu", "sm100.cuh", "common.cuh", "schedule.cuh")


def kernel_source_hash() -> str:
    """Hash of the decode kernel's sources (its file and the device headers it
    includes): a stored ncu traffic figure is only reported while the kernel it
    was taken from is unchanged."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mla_latent_kv_25_b200", "csrc")
    for f in DECODE_KERNEL_SOURCES:
        h.update(f.encode())
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def stored_traffic(workload: str):
    """Per-launch DRAM bytes of the decode kernel from the committed ncu
    summary (profiles/traffic_<workload>.txt: 'kernel_hash <h>' and
    'dram_bytes_per_launch <n>' lines), or None when absent or stale."""
    p = os.path.join(ROOT, "profiles", f"traffic_{workload}.txt")
    if not os.path.exists(p):
        return None
    kv = {}
    for line in open(p):
        parts = line.split()
        if len(parts) >= 2:
            kv[parts[0]] = parts[1]
    if kv.get("kernel_hash") != kernel_source_hash():
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        """Start nvidia-smi and return once its first sample has arrived, so
        that the samples cover the timed region that follows."""
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        first = threading.Event()

        def reader():
            for line in self.proc.stdout:
                if line.strip():
                    self.lines.append(line)
                    first.set()
            first.set()

        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()
        first.wait(timeout=10.0)
        self.lines.clear()  # keep only samples taken from here on

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            self.proc.wait()
        self.thread.join(timeout=5)
        out = "".join(self.lines)
        rows = [r.split(",") for r in out.strip().splitlines() if r.strip()]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)),
                "reasons": sorted(reasons), "samples": len(sm)}


def nvtx_push(name: str):
    """Named range for a profiler timeline (around whole regions, never per step)."""
    try:
        torch.cuda.nvtx.range_push(name)
    except Exception:  # no NVTX library: the ranges are optional
        pass


def nvtx_pop():
    try:
        torch.cuda.nvtx.range_pop()
    except Exception:
        pass


def step_bytes_flops(w):
    dec_b = layout.decode_algorithmic_bytes(w.total_tokens, w.B, w.H, w.cache_dtype,
                                            num_blocks_read=int(((w.seq_lens + 63) // 64).sum()))
    abs_b = layout.absorb_algorithmic_bytes(w.B, w.H)
    dec_f = layout.decode_flops(w.total_tokens, w.H)
    abs_f = layout.absorb_flops(w.B, w.H)
    return dec_b, abs_b, dec_f, abs_f


def time_launches(fn, n: int, stream):
    """Per-launch device times (ms) of ``n`` back-to-back calls of ``fn``,
    each bracketed by CUDA events recorded on ``stream`` (the stream the
    kernels are launched on)."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n)]
    torch.cuda.synchronize()
    for a, b in ev:
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def roofline_block(dec_b: int, dec_f: int, ms_list, peaks: dict, src: str, kernel: str,
                   traffic=None, launches: int = 0) -> dict:
    """Roofline of one decode call: the slower of its algorithmic bytes at the
    measured HBM copy bandwidth and its FLOPs at the measured dense bf16 peak
    (burst: the call is timed on its own); achieved = algorithmic units over
    the mean CUDA-event duration of the call."""
    hbm = float(peaks["hbm_gbs"])
    tens = float(peaks["bf16_tflops"])
    ms = float(np.mean(ms_list))
    t_hbm = dec_b / (hbm * 1e9)
    t_tc = dec_f / (tens * 1e12)
    if t_hbm >= t_tc:
        achieved = dec_b / (ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4)}
    else:
        achieved = dec_f / (ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": tens,
                "unit": "TFLOP/s", "frac": round(achieved / tens, 4)}
    roof.update({
        "traffic": traffic, "algorithmic_bytes": int(dec_b), "flops": int(dec_f),
        "kernel": kernel, "launches_timed": len(ms_list), "kernels_per_call": launches,
        "ms_per_launch": round(ms, 5),
        "ms_per_launch_median": round(float(np.median(ms_list)), 5),
        "ms_per_launch_min": round(float(np.min(ms_list)), 5),
        "roofline_ms": round(max(t_hbm, t_tc) * 1e3, 5),
        "achieved_gbs": round(dec_b / (ms * 1e-3) / 1e9, 1),
        "achieved_tflops": round(dec_f / (ms * 1e-3) / 1e12, 1),
        "peak_source": f"{src} ({'MEASURED_PEAKS.json' if src == 'measured' else 'fallback'})",
    })
    return roof


def decode_kernels_per_call(fp8: bool) -> int:
    """Kernels one mla_decode call launches: the decode kernel and the merge
    (an fp8 cache adds its widening kernel)."""
    return 3 if fp8 else 2


def fp8_through_writers(binding, name: str, dev, stream):
    """The fp8 workload built the way a serving stack fills its cache: the
    seeded rows (c_kv and the key before rotation) are appended through
    mla_cache_append (RoPE in fp32, bf16 rows) and every block is converted
    by mla_cache_quantize_fp8 (per-block scale, E4M3 codes).  Returns the
    workload (its bf16 draws) and the device tensors of the fp8 cache."""
    w = inputs.make(name, cache="bf16")
    d = binding.to_device(w, dev)
    raw = d["cache"]
    nb = ((w.seq_lens.to(torch.int64) + 63) // 64)
    tok_b = torch.repeat_interleave(torch.arange(w.B), w.seq_lens.to(torch.int64))
    starts = torch.cumsum(w.seq_lens.to(torch.int64), 0) - w.seq_lens.to(torch.int64)
    tok_p = torch.arange(int(w.seq_lens.sum())) - torch.repeat_interleave(starts, w.seq_lens.to(torch.int64))
    phys = w.block_table[tok_b, tok_p // 64].to(torch.int64)
    rows = raw[phys.to(dev), (tok_p % 64).to(dev)]                # [T, 576] draws
    c_kv = rows[:, :512].contiguous()
    k_r = rows[:, 512:].contiguous()
    cache_bf16 = torch.zeros_like(raw)
    binding.mla_cache_append(c_kv, k_r, tok_b.to(torch.int32).to(dev), tok_p.to(torch.int32).to(dev),
                             d["block_table"], cache_bf16, stream=stream)
    NB = int(raw.shape[0])
    codes = torch.empty((NB, 64, 512), dtype=torch.uint8, device=dev)
    k_rope = torch.empty((NB, 64, 64), dtype=torch.bfloat16, device=dev)
    scale = torch.empty((NB,), dtype=torch.float32, device=dev)
    binding.mla_cache_quantize_fp8(cache_bf16, torch.arange(NB, dtype=torch.int32, device=dev),
                                   codes, k_rope, scale, stream=stream)
    if binding.mla_cache_get_error(stream) != 0:
        raise RuntimeError("device error in the cache writers")
    del rows, c_kv, k_r, cache_bf16, raw
    d["cache"], d["k_rope"], d["block_scale"] = codes, k_rope, scale
    assert int(nb.sum()) <= NB
    return w, d


def extra_workload(binding, name: str, dev, stream, peaks, src, n_launch: int, num_splits: int):
    """Decode-only timing of another configuration (absorbed queries as
    drawn), with its own roofline block."""
    if name == "fp8":
        w, d = fp8_through_writers(binding, name, dev, stream)
        fp8 = True
        kind = "fp8"
    else:
        w = inputs.make(name)
        d = binding.to_device(w, dev)
        fp8 = False
        kind = w.cache_dtype
    B, H = w.B, w.H
    out = torch.empty((B, H, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    ws = binding.alloc_workspace(B, H, num_splits, device=dev,
                                 fp8_max_blocks=int(w.block_table.shape[1]) if fp8 else None)

    def call():
        binding.mla_decode(d["q"], d["cache"], d["block_table"], d["seq_lens"], w.softmax_scale, out,
                           lse, ws, k_rope=d["k_rope"], block_scale=d["block_scale"],
                           num_splits=num_splits, stream=stream)

    for _ in range(5):
        call()
    ms = time_launches(call, n_launch, stream)
    if binding.mla_get_device_error(ws, stream) != 0:
        raise RuntimeError(f"device error in the {name} decode")
    nblk = int(((w.seq_lens + 63) // 64).sum())
    dec_b = layout.decode_algorithmic_bytes(w.total_tokens, B, H, kind, num_blocks_read=nblk)
    dec_f = layout.decode_flops(w.total_tokens, H)
    roof = roofline_block(dec_b, dec_f, ms, peaks, src,
                          "mla_decode" + (" (fp8 cache)" if fp8 else ""),
                          traffic=stored_traffic(name), launches=decode_kernels_per_call(fp8))
    roof["description"] = inputs.DESCRIPTIONS[name] + (
        "; cache built by mla_cache_append (RoPE in fp32) + mla_cache_quantize_fp8" if fp8 else "")
    roof["tokens"] = w.total_tokens
    del d, out, lse, ws
    torch.cuda.empty_cache()
    return roof


def run_ours(args, world, rank, local):
    from mla_latent_kv_25_b200 import binding

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    w = inputs.make(args.workload, seed=rank_seed(args.workload, rank))
    d = binding.to_device(w, dev)
    B, H = w.B, w.H
    stream = torch.cuda.current_stream(dev)
    q = torch.empty((B, H, 576), dtype=torch.bfloat16, device=dev)
    q_rope = w.q[:, :, 512:].contiguous().to(dev)
    out = torch.empty((B, H, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    fp8 = w.cache_dtype != "bf16"
    ws = binding.alloc_workspace(B, H, args.num_splits, device=dev,
                                 fp8_max_blocks=int(w.block_table.shape[1]) if fp8 else None)
    launches_per_step = 1 + decode_kernels_per_call(fp8)
    dec_b, abs_b, dec_f, abs_f = step_bytes_flops(w)
    peaks, src = load_peaks()

    def decode(qq=None, oo=None, ll=None):
        binding.mla_decode(q if qq is None else qq, d["cache"], d["block_table"], d["seq_lens"],
                           w.softmax_scale, out if oo is None else oo, lse if ll is None else ll,
                           ws, k_rope=d["k_rope"], block_scale=d["block_scale"],
                           num_splits=args.num_splits, stream=stream)

    def step():
        binding.mla_absorb_q(d["q_nope"], d["w_uk"], q_rope, q, stream=stream)
        decode()

    W = max(3, args.warmup)
    nvtx_push("warm-up")
    for _ in range(W):
        step()
    torch.cuda.synchronize(dev)
    nvtx_pop()
    if binding.mla_get_device_error(ws, stream) != 0:
        raise RuntimeError("device error during warm-up")

    clocks = ClockSampler(local)
    clocks.start()
    # device-timed region: exactly K steps between a barrier + synchronize on
    # each side
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    nvtx_push("timed steps")
    t0.record(stream)
    for _ in range(K):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    nvtx_pop()
    if world > 1:
        torch.distributed.barrier()
    ms = t0.elapsed_time(t1)

    # the dominant call, timed on its own over many back-to-back launches
    n_dec = max(200, K)
    nvtx_push("decode launches")
    dec_list = time_launches(decode, n_dec, stream)
    nvtx_pop()
    dec_ms = float(np.mean(dec_list))

    # end to end through the public API with host buffers, as a serving loop
    # runs it: every step copies its new queries (q_nope, q_rope) host->device
    # and its out/lse device->host; inputs and outputs are double-buffered and
    # the copies run on their own streams, so step i+1's upload and step i's
    # download overlap step i's compute.  All copies lie inside the timed
    # region; a few untimed steps of the same loop come first.
    h_qn = w.q_nope.pin_memory()
    h_qr = w.q[:, :, 512:].contiguous().pin_memory()
    h_out = [torch.empty((B, H, 512), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h_lse = [torch.empty((B, H), dtype=torch.float32).pin_memory() for _ in range(2)]
    d_qn = [d["q_nope"], torch.empty_like(d["q_nope"])]
    d_qr = [q_rope, torch.empty_like(q_rope)]
    d_q = [q, torch.empty_like(q)]
    d_out = [out, torch.empty_like(out)]
    d_lse = [lse, torch.empty_like(lse)]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_loop(n):
        ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of buffer k uploaded
        ev_done = [torch.cuda.Event() for _ in range(2)]   # step on buffer k computed
        ev_out = [torch.cuda.Event() for _ in range(2)]    # results of buffer k downloaded
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        up.wait_event(e0)
        down.wait_event(e0)
        for i in range(n):
            k = i & 1
            if i >= 2:
                up.wait_event(ev_done[k])          # step i-2 has read input buffer k
            with torch.cuda.stream(up):
                d_qn[k].copy_(h_qn, non_blocking=True)
                d_qr[k].copy_(h_qr, non_blocking=True)
            ev_in[k].record(up)
            stream.wait_event(ev_in[k])
            if i >= 2:
                stream.wait_event(ev_out[k])       # step i-2's results have left buffer k
            binding.mla_absorb_q(d_qn[k], d["w_uk"], d_qr[k], d_q[k], stream=stream)
            decode(d_q[k], d_out[k], d_lse[k])
            ev_done[k].record(stream)
            down.wait_event(ev_done[k])
            with torch.cuda.stream(down):
                h_out[k].copy_(d_out[k], non_blocking=True)
                h_lse[k].copy_(d_lse[k], non_blocking=True)
            ev_out[k].record(down)
        for k in range(min(2, n)):
            stream.wait_event(ev_out[k])
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / n

    e2e_loop(W)                        # untimed: first copies on fresh streams and buffers
    K2 = max(200, K)
    nvtx_push("end-to-end steps")
    e2e_ms = e2e_loop(K2)
    nvtx_pop()
    clk = clocks.stop()

    # the step after the hot path, timed on its own (not part of the step):
    # output absorption out_h = W_UV[h] . o_latent on this step's output
    o_heads = torch.empty((B, H, 128), dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        binding.mla_absorb_o(out, d["w_uv"], o_heads, stream=stream)
    absorb_o_ms = float(np.mean(time_launches(
        lambda: binding.mla_absorb_o(out, d["w_uv"], o_heads, stream=stream), 200, stream)))
    if binding.mla_absorb_get_error(stream) != 0:
        raise RuntimeError("device error in the output absorption")

    # multi-token decode at the workload's H, timed on its own: q_len draft
    # tokens of H heads per sequence (token 0 = this step's queries, the
    # others seeded normal draws with the queries' spread), causal among the drafts;
    # q_len * H rows above 128 run in 128-row tiles, one cache pass each
    multi = None
    if not fp8 and H == 128:
        multi = []
        gen = torch.Generator().manual_seed(1234)
        for q_len in (2, 4):
            extra = (torch.randn((B, q_len - 1, H, 576), generator=gen) * float(q.float().std())).to(torch.bfloat16)
            qm = torch.cat([q.view(B, 1, H, 576), extra.to(dev)], dim=1).contiguous()
            outm = torch.empty((B, q_len, H, 512), dtype=torch.bfloat16, device=dev)
            lsem = torch.empty((B, q_len, H), dtype=torch.float32, device=dev)
            wsm = binding.alloc_workspace(B, q_len * H, args.num_splits, device=dev)

            def mcall(qm=qm, outm=outm, lsem=lsem, wsm=wsm):
                binding.mla_decode_multi(qm, d["cache"], d["block_table"], d["seq_lens"],
                                         w.softmax_scale, outm, lsem, wsm, num_splits=args.num_splits,
                                         stream=stream)
            for _ in range(3):
                mcall()
            m_ms = float(np.mean(time_launches(mcall, 50, stream)))
            if binding.mla_get_device_error(wsm, stream) != 0:
                raise RuntimeError("device error in the multi-token decode")
            mb = layout.decode_algorithmic_bytes(w.total_tokens, B, q_len * H, "bf16")
            mf = layout.decode_flops(w.total_tokens, q_len * H)
            t_hbm = mb / (float(peaks["hbm_gbs"]) * 1e9) * 1e3
            t_tc = mf / (float(peaks["bf16_tflops"]) * 1e12) * 1e3
            multi.append({"q_len": q_len, "heads_per_token": H, "rows_per_sequence": q_len * H,
                          "cache_passes": (q_len * H + 127) // 128,
                          "ms_per_launch": round(m_ms, 5), "algorithmic_bytes": mb, "flops": mf,
                          "bound": "tensor" if t_tc > t_hbm else "hbm",
                          "roofline_ms": round(max(t_hbm, t_tc), 5),
                          "frac": round(max(t_hbm, t_tc) / m_ms, 4)})
            del qm, outm, lsem, wsm
    if binding.mla_get_device_error(ws, stream) != 0:
        raise RuntimeError("device error during timing")

    step_ms = ms / K
    step_ms, dec_ms, e2e_ms = max_over_ranks([step_ms, dec_ms, e2e_ms], dev)

    extras = {}
    if world == 1 and args.workload == "v3" and not args.no_extra_workloads:
        del ws
        for name in ("ragged", "long", "fp8"):
            extras[name] = extra_workload(binding, name, dev, stream, peaks, src, 100,
                                          args.num_splits)

    res = None
    if rank == 0:
        step_bytes = dec_b + abs_b
        value = job_rate(step_bytes, world, step_ms)
        roof = roofline_block(dec_b, dec_f, dec_list, peaks, src,
                              "mla_decode" + (" (fp8 cache)" if fp8 else ""),
                              traffic=stored_traffic(args.workload),
                              launches=decode_kernels_per_call(fp8))
        if world > 1:
            roof["ms_per_launch_max_over_ranks"] = round(dec_ms, 5)
        res = {
            "metric": METRIC,
            "value": round(value, 1),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": K,
            "warmup": W,
            "ms_per_step": round(step_ms, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16" if w.cache_dtype == "bf16" else "fp8-e4m3 cache, bf16 mma",
            "data": "synthetic (seeded; DeepSeek-V3 decode shape, random-permuted paged cache)",
            "config": {"workload": args.workload, "description": inputs.DESCRIPTIONS[args.workload],
                       "B": B, "H": H, "tokens": w.total_tokens, "cache": w.cache_dtype,
                       "num_splits": args.num_splits,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "inputs larger than L2 (cache %.0f MB > 126 MB); no flush"
                             % (w.cache.numel() * w.cache.element_size() / 1e6)},
            "tflops": round((dec_f + abs_f) * world / (step_ms * 1e-3) / 1e12, 2),
            "decode_tflops": round(dec_f / (dec_ms * 1e-3) / 1e12, 2),
            "roofline": roof,
            "e2e": {"value": round(job_rate(step_bytes, world, e2e_ms), 1), "unit": "GB/s",
                    "ms_per_step": round(e2e_ms, 5), "steps": K2,
                    "h2d_bytes_per_step": int(h_qn.numel() * 2 + h_qr.numel() * 2),
                    "d2h_bytes_per_step": int(h_out[0].numel() * 2 + h_lse[0].numel() * 4),
                    "pipelined": "double-buffered; copies on their own streams overlap compute"},
            "gpu_launches": launches_per_step * K,
            "absorb_o": absorb_o_line(B, H, absorb_o_ms, float(peaks["hbm_gbs"])),
            "multi_token": multi,
            "workloads": extras or None,
            "clocks": clk,
        }
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return res, w


def oracle_sample_rate(w, seconds: float, n_seq_max=None):
    """Time the oracle on whole sequences of the workload until ~``seconds``
    of work; returns (GB/s of algorithmic bytes, threads, description)."""
    import oracle
    cores = oracle.max_threads()
    done_tokens = 0
    rows = 0
    t_total = 0.0
    b = 0
    # at least one whole sequence, whatever the time budget
    while b < w.B and (b == 0 or t_total < seconds) and (n_seq_max is None or b < n_seq_max):
        units = np.stack([np.full(w.H, b), np.arange(w.H), np.zeros(w.H), -np.ones(w.H)], 1)
        t = time.perf_counter()
        oracle.decode_units(q=w.q, cache=w.cache, block_table=w.block_table, seq_lens=w.seq_lens,
                            num_blocks=w.num_blocks, softmax_scale=w.softmax_scale,
                            units=units.astype(np.int32), cache_kind=w.cache_dtype,
                            k_rope=w.k_rope, block_scale=w.block_scale)
        t_total += time.perf_counter() - t
        done_tokens += int(w.seq_lens[b])
        rows += w.H
        b += 1
    nb = int((done_tokens + 63) // 64)
    by = layout.decode_algorithmic_bytes(done_tokens, b, w.H, w.cache_dtype, nb)
    desc = f"{b} of {w.B} sequences x {w.H} heads ({done_tokens} tokens) of workload {w.name}"
    return by / t_total / 1e9, cores, desc, t_total


def run_reference(args, world, rank):
    if rank != 0:
        return
    w = inputs.make(args.workload)
    dec_b, abs_b, _, _ = step_bytes_flops(w)
    vals = []
    K = max(1, min(args.steps, 3))
    desc, cores = "", 1
    for _ in range(max(0, min(args.warmup, 1))):
        oracle_sample_rate(w, 0.0, n_seq_max=1)
    per = max(1.0, args.cpu_seconds / K)
    for _ in range(K):
        v, cores, desc, _t = oracle_sample_rate(w, per)
        vals.append(v)
    v = float(np.median(vals))
    ms = (dec_b + abs_b) / (v * 1e9) * 1e3
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s",
            "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": round(ms, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)",
            "config": {"workload": args.workload, "description": inputs.DESCRIPTIONS[args.workload]},
            "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": desc + " per step"},
            "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    emit(line, args.json_out)


def emit(line: dict, path=None):
    """Print the one JSON result line (and append it to ``path`` if given)."""
    text = json.dumps(line)
    print(text, flush=True)
    if path:
        with open(path, "a") as f:
            f.write(text + "\n")


def main():
    args = parse()
    world, rank, local = dist_env()
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    res, w = run_ours(args, world, rank, local)
    if rank == 0:
        if not args.no_cpu_baseline and world == 1:
            v, cores, desc, t = oracle_sample_rate(w, args.cpu_seconds)
            res["cpu_baseline"] = {"value": round(v, 4), "unit": "GB/s", "cores": cores,
                                   "kind": "oracle", "sample": desc + f", {t:.1f} s"}
        emit(res, args.json_out)


if __name__ == "__main__":
    main()
