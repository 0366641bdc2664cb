"""Benchmark: block-causal chunk attention over a Wan2.1-1.3B-shaped 5-step wavefront.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {wf,reference}] [--workload W]

One step is one pass of the whole hot path over one layer of the wavefront: wf_kv_append of the
five active chunks' K/V into their pages (the two clean context chunks are appended once, before
timing) and one wf_attn_forward over all chunks.  Inputs are seeded synthetic tensors of the
workload's shapes, resident in HBM before the timed region (q 72 MB, K/V 144 MB appended per step,
201 MB of K/V pages read, 72 MB written: far larger than the 126 MB L2).

Printed (rank 0, one JSON line): throughput in TFLOP/s of algorithmic attention work
(4 * D * H * sum over query rows of visible keys; masked pairs, exp and rescaling not counted),
with tokens/s, the roofline of the attention kernel, an end-to-end figure through the C ABI with
host buffers, the CPU oracle as a baseline, and the SM clocks seen during the timed region.

--workload wan13b_4step / wan14b run the other full-size wavefronts; --workload wp_rank0 runs one
Wave-Parallelism rank's call (one 4680-token chunk against a 37 440-key prefix) through
wf_attn_forward_split with the library's choice of key splits, whose timed attention then
includes the merge kernel.

With --gpus N > 1 (launched by torch.distributed.run) every rank runs an independent replica of
the same workload: the path has no exchange step, so there is no data-path collective; a barrier
and a max-reduction of the device times are the only collectives.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_causal_streaming_b200.workloads import (WORKLOADS, WP_RANK0, Workload,  # noqa: E402
                                                   make_inputs)

METRIC = "block-causal chunk-attention TFLOP/s and % of B200 bf16 peak; tokens/s"
UNIT = "TFLOP/s"
# the attention kernel and the host code that sets up its launch (tensor-map boxes, grid order)
KERNEL_SOURCES = ["block_causal_streaming_b200/csrc/attn_kernel.cuh",
                  "block_causal_streaming_b200/csrc/sm100.cuh",
                  "block_causal_streaming_b200/csrc/wf_api.cu"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------------------ accounting
BENCH_WORKLOADS = ("wan13b_5step", "wan13b_4step", "wan14b", "wp_rank0")


def workload_of(name: str) -> Workload:
    return WORKLOADS[name]


def attention_flops(wl: Workload) -> int:
    """4 * D * H * sum over query rows of the number of keys that row may see."""
    off, nctx = wl.chunk_offsets, wl.num_ctx_chunks
    visible = sum((off[c + 1] - off[c]) * off[c + 1] for c in range(nctx, wl.num_chunks))
    return 4 * wl.head_dim * wl.heads * visible


def rows_flops(wl: Workload, rows, heads_per_row: int) -> int:
    off, nctx = wl.chunk_offsets, wl.num_ctx_chunks
    t_ctx = off[nctx]
    total = 0
    for r in rows:
        t = t_ctx + r
        c = next(i for i in range(wl.num_chunks) if off[i] <= t < off[i + 1])
        total += off[c + 1]
    return 4 * wl.head_dim * heads_per_row * total


def workload_config(wl: Workload, world: int, split: bool) -> dict:
    """The `config` object of a bench line: the workload, with its sizes, and how a step runs.
    Both arms print the same object for the same workload."""
    off, nctx = wl.chunk_offsets, wl.num_ctx_chunks
    H, D = wl.heads, wl.head_dim
    active = wl.num_chunks - nctx
    # q, out, the appended K/V (read + written) and the K/V pages attention reads
    touched_mb = (2 * wl.t_q * H * D + 4 * (off[-1] - off[nctx]) * H * D + 2 * off[-1] * H * D) \
        * 2 / 1e6
    return {"workload": wl.name, "heads": H, "head_dim": D, "t_q": wl.t_q, "t_kv": wl.t_kv,
            "chunks": f"{nctx} ctx + {active} active x {off[nctx + 1] - off[nctx]}",
            "page_size": wl.page_size,
            "step": f"append {active} active chunks + attention"
                    + (" (key splits + merge)" if split else ""),
            "l2": f"inputs larger than L2 (~{touched_mb:.0f} MB touched per step vs 126 MB L2)",
            "parallelism": f"replicas x{world}"}


def kernel_hash() -> str:
    """Hash of the attention sources' code: comments and blank space removed, so that an edit of
    a comment keeps a traffic record valid and any change of code drops it."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)       # block comments
        text = re.sub(r"//[^\n]*", " ", text)                     # line comments
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def load_traffic(workload: str):
    """DRAM bytes per attention launch from a committed ncu capture, if it matches this kernel
    and workload."""
    path = os.path.join(ROOT, "profiles", "attn_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("kernel_hash") != kernel_hash() or rec.get("workload") != workload:
        return None
    return rec.get("dram_bytes_per_launch")


# ------------------------------------------------------------------------------ distributed
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(backend=backend,
                                             timeout=datetime.timedelta(seconds=120))


def barrier(world: int, device=None):
    if world > 1:
        if device is not None and torch.distributed.get_backend() == "nccl":
            torch.distributed.barrier(device_ids=[device.index])
        else:
            torch.distributed.barrier()


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64,
                     device=device if torch.distributed.get_backend() == "nccl" else "cpu")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate(units_per_rank: float, world: int, seconds_max: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / seconds_max


# ------------------------------------------------------------------------------ clocks
class ClockSampler:
    """NVML samples (every 10 ms, read-only) of SM clock, power and clock-event reasons while
    the timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device: torch.device):
        self.device = device
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        self._nvml = pynvml
        try:
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
        except Exception:  # fall back to the visible-device index
            idx = self.device.index or 0
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            if vis:
                idx = int(vis.split(",")[idx])
            return pynvml.nvmlDeviceGetHandleByIndex(idx)

    def _run(self, h):
        nv = self._nvml
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetPowerUsage(h) / 1000.0, int(get_reasons(h))))
            except Exception:
                pass
            self._stop.wait(0.01)

    def __enter__(self):
        try:
            h = self._handle()
            self.max_mhz = self._nvml.nvmlDeviceGetMaxClockInfo(h, self._nvml.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._run, args=(h,), daemon=True)
            self._thread.start()
            t0 = time.time()
            while not self.samples and time.time() - t0 < 2.0:
                time.sleep(0.005)
        except Exception:
            self._thread = None
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"],
                    "samples": 0}
        reasons = sorted({name for _, _, r in self.samples for bit, name in self.REASONS.items()
                          if r & bit})
        return {"sm_mhz": statistics.median(c for c, _, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples),
                "power_w_max": round(max(pw for _, pw, _ in self.samples), 1)}


# ------------------------------------------------------------------------------ CPU oracle
def oracle_sample(wl: Workload, inp, target_s: float, seed: int = 0):
    """Time the oracle on a bounded sample of query rows (all heads); returns (TFLOP/s, info)."""
    import oracle  # CPU-baseline leg only
    rng = np.random.default_rng(seed)
    q32 = inp.q.float().numpy()
    k32 = inp.k.float().numpy()
    v32 = inp.v.float().numpy()
    scale = 1.0 / np.sqrt(wl.head_dim)
    H = wl.heads
    threads = oracle.default_threads()

    def run(rows):
        rr = np.repeat(np.asarray(rows, dtype=np.int32), H)
        hh = np.tile(np.arange(H, dtype=np.int32), len(rows))
        t0 = time.perf_counter()
        oracle.attention_rows(q32, k32, v32, wl.chunk_offsets, wl.num_ctx_chunks, scale, rr, hh,
                              nthreads=threads)
        return time.perf_counter() - t0

    probe = sorted(rng.choice(wl.t_q, size=4, replace=False).tolist())
    t_probe = run(probe)
    per_row = t_probe / len(probe)
    n = int(max(4, min(wl.t_q, target_s / max(per_row, 1e-6))))
    rows = sorted(rng.choice(wl.t_q, size=n, replace=False).tolist())
    dt = run(rows)
    fl = rows_flops(wl, rows, H)
    info = {"rows": n, "heads": H, "seconds": round(dt, 3), "flop": fl, "threads": threads}
    return fl / dt / 1e12, info


# ------------------------------------------------------------------------------ GPU arm
def fp8_kv_leg(wl: Workload, layer, k, v, dev, stream, steps: int, warmup: int,
               hbm_peak: float) -> dict:
    """The FP8 transport kernels over every chunk of the workload's layer: wf_kv_append_fp8
    (bf16 rows -> e4m3 pages + per-(token, head) scales) and wf_kv_dequant (back into the bf16
    pool), one launch per chunk as a Wave-Parallelism producer and consumer run them, and the
    chunk-range forms (wf_kv_append_fp8_chunks / wf_kv_dequant_chunks) over the whole layer in
    one launch each.  Each leg is timed with CUDA events on the launching stream after a 256 MB
    read that evicts L2; the read writes back whatever the previous leg left dirty, outside the
    timed region, and leaves L2 holding clean lines only.  Algorithmic bytes: every K/V element
    read once in one format and written once in the other."""
    import block_causal_streaming_b200 as wf
    from block_causal_streaming_b200.layer import PagedPoolFp8
    H, D, off = wl.heads, wl.head_dim, wl.chunk_offsets
    fp = PagedPoolFp8(wl.num_pages, wl.page_size, H, D, dev)
    flush = torch.ones(64 * 2 ** 20, dtype=torch.float32, device=dev)       # 256 MB > L2
    sink = torch.empty((), dtype=torch.float32, device=dev)
    chunks = range(wl.num_chunks)

    def quant():
        for c in chunks:
            wf.kv_append_fp8(*fp.tensors, 0, c, k[off[c]:off[c + 1]], v[off[c]:off[c + 1]],
                             layer.page_tables, layer.desc, stream)

    def dequant():
        for c in chunks:
            wf.kv_dequant(*fp.tensors, layer.pool.k, layer.pool.v, 0, c, layer.page_tables,
                          layer.desc, stream)

    def append_bf16():
        layer.append_range(k, v, chunks, stream)

    def quant_range():
        wf.kv_append_fp8_chunks(*fp.tensors, 0, 0, wl.num_chunks, k, v, layer.page_tables,
                                layer.desc, stream)

    def dequant_range():
        wf.kv_dequant_chunks(*fp.tensors, layer.pool.k, layer.pool.v, 0, 0, wl.num_chunks,
                             layer.page_tables, layer.desc, stream)

    legs = (quant, dequant, append_bf16, quant_range, dequant_range)
    for _ in range(warmup):
        for leg in legs:
            leg()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * len(legs))]
           for _ in range(steps)]
    torch.cuda.synchronize(dev)
    for e in evs:
        for i, leg in enumerate(legs):
            torch.sum(flush, dim=(0,), out=sink)
            e[2 * i].record(stream)
            leg()
            e[2 * i + 1].record(stream)
    torch.cuda.synchronize(dev)
    rc = wf.check_status()
    if rc != wf.WF_OK:
        raise RuntimeError(f"device status after the FP8 leg: {wf.strerror(rc)}")
    rows = off[-1]
    elems = 2 * rows * H * D                      # K and V
    bf16_bytes, fp8_bytes = 2 * elems, elems + 2 * rows * H * 4
    out = {"chunks": wl.num_chunks, "tokens": rows, "steps": steps,
           "bytes_bf16": bf16_bytes, "bytes_fp8": fp8_bytes,
           "bytes_ratio": round(fp8_bytes / bf16_bytes, 4), "peak_gbs": hbm_peak}
    # the plain bf16 append of the same chunks, timed the same way: what one launch per chunk
    # of this size reaches for a pure copy
    for name, (a, b), nbytes, launches in (
            ("append_fp8", (0, 1), bf16_bytes + fp8_bytes, wl.num_chunks),
            ("dequant", (2, 3), bf16_bytes + fp8_bytes, wl.num_chunks),
            ("append_bf16_reference", (4, 5), 2 * bf16_bytes, wl.num_chunks),
            ("append_fp8_one_launch", (6, 7), bf16_bytes + fp8_bytes, 1),
            ("dequant_one_launch", (8, 9), bf16_bytes + fp8_bytes, 1)):
        ms = statistics.mean(e[a].elapsed_time(e[b]) for e in evs)
        gbs = nbytes / (ms / 1e3) / 1e9
        out[name] = {"ms": round(ms, 4), "gbs": round(gbs, 1), "frac": round(gbs / hbm_peak, 4),
                     "launches": launches}
    return out


def int8_leg(wl: Workload, layer, q, dev, stream, steps: int, warmup: int, peak: float,
             out_bf16, fmt: str = "int8") -> dict:
    """An 8-bit QK^T attention tier on the workload's layer -- fmt "int8": wf_qk_quantize_i8 (key
    mean, int8 codes and scales of K' and Q) and wf_attn_forward_i8; "e4m3": wf_qk_quantize_e4m3
    and wf_attn_forward_e4m3 -- each timed with CUDA events on the launching stream; TFLOP/s on
    the same algorithmic FLOP count as the bf16 path.  `out_bf16`: the bf16 path's output, for
    the tier's deviation from it."""
    import block_causal_streaming_b200 as wf
    from block_causal_streaming_b200.layer import QkE4m3Buffers, QkI8Buffers
    e4m3 = fmt == "e4m3"
    qk = (QkE4m3Buffers if e4m3 else QkI8Buffers)(layer.desc, wl.heads, wl.head_dim, dev)
    out = torch.empty_like(q)
    row = layer.page_tables[layer.layer]
    scale = 1.0 / np.sqrt(wl.head_dim)
    quantize = wf.qk_quantize_e4m3 if e4m3 else wf.qk_quantize_i8
    forward = wf.attn_forward_e4m3 if e4m3 else wf.attn_forward_i8

    def quant():
        quantize(q, layer.pool.k, layer.pool.v, row, layer.desc, qk, stream)

    def attn():
        forward(qk, layer.pool.k, layer.pool.v, row, layer.desc, scale, out, None, stream)

    for _ in range(warmup):
        quant()
        attn()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    torch.cuda.synchronize(dev)
    for e in evs:
        e[0].record(stream)
        quant()
        e[1].record(stream)
        attn()
        e[2].record(stream)
    torch.cuda.synchronize(dev)
    rc = wf.check_status()
    if rc != wf.WF_OK:
        raise RuntimeError(f"device status after the {fmt} leg: {wf.strerror(rc)}")
    q_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    a_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    flop = attention_flops(wl)
    dev_abs = (out.float() - out_bf16.float()).abs()
    return {"steps": steps, "quantize_ms": round(q_ms, 4), "attn_ms": round(a_ms, 4),
            "attn_tflops": round(flop / (a_ms / 1e3) / 1e12, 2),
            "frac_of_bf16_peak": round(flop / (a_ms / 1e3) / 1e12 / peak, 4),
            "vs_bf16_output": {"max_abs": round(float(dev_abs.max()), 5),
                               "mean_abs": round(float(dev_abs.mean()), 6)}}


def gpu_arm(args, world, rank, local):
    import block_causal_streaming_b200 as wf
    from block_causal_streaming_b200.layer import PagedPool, WavefrontLayer

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    wl = workload_of(args.workload)
    inp = make_inputs(wl)
    H, D = wl.heads, wl.head_dim
    off, nctx = wl.chunk_offsets, wl.num_ctx_chunks
    scale = 1.0 / np.sqrt(D)
    flop = attention_flops(wl)

    pool = PagedPool(wl.num_pages, wl.page_size, H, D, dev)
    pt = inp.page_table.to(dev).reshape(1, -1).contiguous()
    layer = WavefrontLayer(pool, pt, 0, off, wl.chunk_stage, nctx)
    q = inp.q.to(dev)
    k = inp.k.to(dev)
    v = inp.v.to(dev)
    out = torch.empty_like(q)
    active = list(range(nctx, wl.num_chunks))
    layer.append_range(k, v, range(nctx))            # clean context: published once
    stream = torch.cuda.current_stream(dev)
    splits = 0 if wl is WP_RANK0 else None            # library-chosen key splits
    split_used = splits is not None and wf.attn_workspace_size(layer.desc, H, D, 0) > 0
    launches_per_step = len(active) + 1 + (1 if split_used else 0)

    def step(ev_pair=None):
        layer.append_range(k, v, active)
        if ev_pair is not None:
            ev_pair[0].record(stream)
        layer.forward(q, out, scale=scale, splits=splits)
        if ev_pair is not None:
            ev_pair[1].record(stream)

    for _ in range(args.warmup):
        step()
    rc = wf.check_status()
    if rc != wf.WF_OK:
        raise RuntimeError(f"device status after warm-up: {wf.strerror(rc)}")

    # ---- timed region: K steps, device time by CUDA events on the launching stream
    attn_events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clocks:
        barrier(world, dev)
        torch.cuda.synchronize(dev)
        t_start.record(stream)
        for i in range(args.steps):
            step(attn_events[i])
        t_stop.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world, dev)
    elapsed = t_start.elapsed_time(t_stop) / 1e3
    attn_ms = [a.elapsed_time(b) for a, b in attn_events]
    elapsed_max = max_over_ranks(elapsed, world, dev)
    rc = wf.check_status()
    if rc != wf.WF_OK:
        raise RuntimeError(f"device status after timing: {wf.strerror(rc)}")

    # ---- end to end through the C ABI with host buffers (pinned), copies inside the region.
    # Every step copies its inputs (q and the active chunks' K/V) host -> device, runs the path
    # and copies the output back.  Three streams overlap step i's compute with the input copy of
    # step i+1 and the output copy of step i-1 (two buffers of each), as a serving loop would.
    q_h = inp.q.pin_memory()
    act_rows = slice(off[nctx], off[-1])
    k_h = inp.k[act_rows].contiguous().pin_memory()
    v_h = inp.v[act_rows].contiguous().pin_memory()
    out_h = [torch.empty(q.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    q_in = [torch.empty_like(q) for _ in range(2)]
    k_act = [torch.empty(k_h.shape, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    v_act = [torch.empty(v_h.shape, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    outs = [torch.empty_like(q) for _ in range(2)]
    h2d = q_h.numel() * 2 + k_h.numel() * 2 + v_h.numel() * 2
    d2h = out_h[0].numel() * 2
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()                                            # noqa: E731
    in_ready, in_free, done, out_free = ([ev(), ev()] for _ in range(4))
    for b in range(2):                       # every buffer starts free
        in_free[b].record(stream)
        out_free[b].record(stream)

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(in_free[b])
            q_in[b].copy_(q_h, non_blocking=True)
            k_act[b].copy_(k_h, non_blocking=True)
            v_act[b].copy_(v_h, non_blocking=True)
            in_ready[b].record(s_in)
        stream.wait_event(in_ready[b])
        stream.wait_event(out_free[b])
        base = off[nctx]
        for c in active:
            lo, hi = off[c] - base, off[c + 1] - base
            layer.append(c, k_act[b][lo:hi], v_act[b][lo:hi], stream)
        layer.forward(q_in[b], outs[b], scale=scale, stream=stream, splits=splits)
        in_free[b].record(stream)
        done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done[b])
            out_h[b].copy_(outs[b], non_blocking=True)
            out_free[b].record(s_out)

    for i in range(max(2, min(args.warmup, 4))):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    e_steps = max(4, min(args.steps, 12))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    e0.record(s_in)
    stream.wait_event(e0)
    for i in range(e_steps):
        e2e_step(i)
    for b in range(2):                       # the region ends when the last output is on the host
        s_in.wait_event(out_free[b])
    e1.record(s_in)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    e_elapsed = max_over_ranks(e0.elapsed_time(e1) / 1e3, world, dev)
    rc = wf.check_status()
    if rc != wf.WF_OK:
        raise RuntimeError(f"device status after end-to-end run: {wf.strerror(rc)}")

    peaks, peak_src = load_peaks()
    step_s = elapsed_max / args.steps
    value = aggregate(flop, world, step_s) / 1e12
    attn_avg_s = statistics.mean(attn_ms) / 1e3
    achieved = flop / attn_avg_s / 1e12
    peak = float(peaks["bf16_tflops"])
    res = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(step_s * 1e3, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1)*0.5 bf16)",
        "config": workload_config(wl, world, split_used),
        "tokens_per_s": round(world * wl.t_q / step_s, 1),
        "pct_of_peak": round(100.0 * value / world / peak, 2),
        "roofline": {"bound": "tensor",
                     "kernel": "wf_attn_fwd_kernel<128>"
                               + (" + wf_combine_kernel<128>" if split_used else ""),
                     "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": load_traffic(wl.name),
                     "peak_source": f"{peak_src} bf16_tflops (burst)",
                     "attn_ms_avg": round(attn_avg_s * 1e3, 4),
                     "attn_ms_p50": round(statistics.median(attn_ms), 4)},
        "e2e": {"value": round(aggregate(flop, world, e_elapsed / e_steps) / 1e12, 2),
                "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e_steps, "overlap": "input copy of step i+1 and output copy of "
                                             "step i-1 run during step i (3 streams)"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks.summary(),
    }
    if args.fp8_kv:
        res["fp8_kv"] = fp8_kv_leg(wl, layer, k, v, dev, stream, max(5, min(args.steps, 20)),
                                   args.warmup, float(peaks["hbm_gbs"]))
    if args.int8 or args.e4m3:
        ref_out = torch.empty_like(q)
        layer.forward(q, ref_out, scale=scale)
        for fmt, on in (("int8", args.int8), ("e4m3", args.e4m3)):
            if not on:
                continue
            if D != 128:
                res[fmt] = {"unavailable": "the 8-bit tiers run head_dim 128"}
            else:
                res[fmt] = int8_leg(wl, layer, q, dev, stream, max(5, min(args.steps, 20)),
                                    args.warmup, peak, ref_out, fmt)
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        tflops, info = oracle_sample(wl, inp, target_s=args.cpu_seconds)
        res["cpu_baseline"] = {"value": round(tflops, 6), "unit": UNIT,
                               "cores": info["threads"], "kind": "oracle",
                               "sample": f"{info['rows']} random query rows x {info['heads']} "
                                         f"heads of the same workload, {info['seconds']} s"}
    if world > 1:
        torch.distributed.barrier(device_ids=[dev.index])
        torch.distributed.destroy_process_group()
    return res


# ------------------------------------------------------------------------------ reference arm
def reference_arm(args, world, rank):
    """The oracle as it stands, on the host cores, on bounded samples of the same workload."""
    if rank != 0:
        return None
    wl = workload_of(args.workload)
    inp = make_inputs(wl)
    per_step = max(1.0, args.cpu_seconds / max(1, args.steps))
    for i in range(args.warmup):
        oracle_sample(wl, inp, target_s=min(per_step, 1.0), seed=1000 + i)
    vals, secs, rows, threads = [], 0.0, 0, 0
    for i in range(args.steps):
        v, info = oracle_sample(wl, inp, target_s=per_step, seed=i)
        threads = info["threads"]
        vals.append(v)
        secs += info["seconds"]
        rows += info["rows"]
    value = statistics.mean(vals)
    sample = f"{args.steps} steps, each a random sample of query rows x {wl.heads} heads " \
             f"({rows} rows, {secs:.1f} s total)"
    return {
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * secs / args.steps, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1)*0.5 bf16)", "impl": "reference",
        "config": workload_config(wl, world, wl is WP_RANK0),
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["wf", "reference"], default="wf")
    ap.add_argument("--workload", default="wan13b_5step", choices=BENCH_WORKLOADS)
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--int8", action="store_true",
                    help="also time the INT8 attention tier (quantize + attention) on the "
                         "workload's layer")
    ap.add_argument("--e4m3", action="store_true",
                    help="also time the FP8 (e4m3) attention tier (quantize + attention)")
    ap.add_argument("--fp8-kv", action="store_true",
                    help="also time the FP8 K/V transport kernels (append to e4m3 pages, "
                         "dequantize) on the workload's chunks")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_env()
    if world != args.gpus and world != 1:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if args.impl == "reference":
        res = reference_arm(args, world, rank)
    else:
        res = gpu_arm(args, world, rank, local)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
