#!/usr/bin/env python
"""Benchmark of the absorbed sparse-MLA decode step (DeepSeek-V3.2-Exp sparse
latent attention, decode branch) on B200.

Workload (default): B=128 decode rows, per-row end_pos uniform in
[4096, 131072], top-k = 2048 positions per row (half from the last 4096
positions, half from the rest), bf16 cache [128, 131072, 576] (19.3 GB),
128 heads.  One step = one ``mla_decode`` call over the batch: fold of W_UK,
gather + scores + softmax + latent mix, split merge + W_UV.

Metric: head*keys/s = (rows x selected keys x 128 heads) per second, summed
over ranks; also microseconds per step.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Under torchrun each rank runs the same per-GPU workload (weak scaling, no
data-path collective); the timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

HEADS = 128
ROW_BYTES = 576 * 2
METRIC = "sparse MLA decode head*keys/s"
UNIT = "head*keys/s"
L2_FLUSH_BYTES = 256 << 20
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "core_kernel_config3_traffic.txt")


# ---------------------------------------------------------------------------
# host-side helpers (importable without a GPU; covered by CPU tests)
# ---------------------------------------------------------------------------

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def algorithmic_work(B: int, k: int):
    """Bytes and flops the method itself must move / compute per step:
    gathered rows + queries + indices + output + wkv_b read once; fold and
    W_UV GEMMs + the two score/mix contractions over the selected keys."""
    bytes_ = B * k * ROW_BYTES + B * (HEADS * 128 * 2 + HEADS * 64 * 2 + 4 * k + HEADS * 128 * 2) \
        + 128 * 256 * 512 * 2
    flops = B * (2 * 2 * HEADS * 128 * 512 + k * 2 * HEADS * (576 + 512))
    return bytes_, flops


def core_kernel_work(B: int, k: int):
    """Algorithmic bytes / flops of the attend kernel alone: each selected
    row (1152 B) and its index (4 B) once; 2*128*(576+512) flops per key."""
    return B * k * (ROW_BYTES + 4), B * k * 2 * HEADS * (576 + 512)


def load_peaks(path=os.path.join(ROOT, "MEASURED_PEAKS.json")):
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def code_only(text):
    """C++/CUDA source without // comments, trailing blanks and empty lines:
    what the compiler sees of it, so that editing a comment does not
    invalidate a profile taken on the same code.  (The sources use no block
    comments, and no string literal in them holds //.)"""
    out = []
    for line in text.splitlines():
        code = line.split("//", 1)[0].rstrip()
        if code:
            out.append(code)
    return "\n".join(out) + "\n"


def kernel_source_sha(texts=None):
    """sha256 of the attend kernel's code (decode.cu and common.cuh, comments
    removed); `texts` may give the two files' contents instead of reading them."""
    h = hashlib.sha256()
    rels = ("sparse_head_latent_absorbed_b200/csrc/decode.cu",
            "sparse_head_latent_absorbed_b200/csrc/common.cuh")
    for i, rel in enumerate(rels):
        if texts is not None:
            text = texts[i]
        else:
            with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
                text = f.read()
        h.update(code_only(text).encode())
    return h.hexdigest()


def profiled_traffic():
    """Per-launch DRAM bytes of the attend kernel from the committed ncu
    summary, or None when that summary is missing or was taken on other
    kernel sources."""
    try:
        kv = {}
        with open(PROFILE_TRAFFIC) as f:
            for line in f:
                if ":" in line:
                    a, b = line.split(":", 1)
                    kv[a.strip()] = b.strip()
        if kv.get("source_sha256") != kernel_source_sha():
            return None
        return float(kv["dram_bytes_per_launch"])
    except Exception:
        return None


def reduce_max(value: float, world: int, device=None) -> float:
    """Max over ranks (a timing reduction, not part of the data path)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons, polled through NVML from a
    background thread every few milliseconds while the timed steps run.

    Only reads the device state; nothing here changes a clock or a limit.
    `wait_live()` returns once the first sample is in, so that a short timed
    region is still covered."""
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, device, period_s: float = 0.005):
        self.device = device
        self.period = period_s
        self.rows = []          # (sm_mhz, max_mhz, reasons bitmask, power_w)
        self.error = None
        self._stop = threading.Event()
        self._live = threading.Event()
        self._thread = None

    def _handle(self, nv):
        import torch
        props = torch.cuda.get_device_properties(self.device)
        try:
            return nv.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid))
        except Exception:
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)

    def _run(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
        except Exception as e:  # no NVML: the line says so
            self.error = f"nvml unavailable: {e}"
            self._live.set()
            return
        try:
            h = self._handle(nv)
            mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            while not self._stop.is_set():
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                try:
                    pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                except Exception:
                    pw = None
                self.rows.append((sm, mx, rs, pw))
                self._live.set()
                self._stop.wait(self.period)
        except Exception as e:
            self.error = f"nvml query failed: {e}"
            self._live.set()
        finally:
            try:
                nv.nvmlShutdown()
            except Exception:
                pass

    def __enter__(self):
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        return self

    def wait_live(self, timeout_s: float = 10.0):
        self._live.wait(timeout_s)

    def mark(self):
        """Index of the next sample: samples from here on fall in the region."""
        return len(self.rows)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=5)

    def summary(self, start: int = 0):
        rows = self.rows[start:]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None,
                    "reasons": [self.error or "no samples"], "samples": 0}
        import pynvml as nv
        reasons = sorted({name for _, _, rs, _ in rows for name, const in self.REASONS
                          if rs & getattr(nv, const, 0)})
        pw = [r[3] for r in rows if r[3] is not None]
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows), "source": "nvml",
                "power_w_median": statistics.median(pw) if pw else None}


# ---------------------------------------------------------------------------
# reference arm: the float64 oracle on the host cores
# ---------------------------------------------------------------------------

def oracle_sample_rate(wl, rows, repeats=1, min_seconds=0.0):
    """Time the oracle (as it stands) on the compacted selected rows of the
    given batch rows, `repeats` passes and then more until `min_seconds` of
    CPU work have run; returns (head*keys/s, seconds, threads, passes)."""
    import numpy as np

    import mla_inputs as mi
    import oracle as orc
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count() or 1
    prepared = []
    for b in rows:
        r, keep = mi.compact_rows(wl, b)
        r = mi.f64(r)
        n = len(keep)
        prepared.append((mi.f64(wl.q_nope[b:b + 1]), mi.f64(wl.q_pe[b:b + 1]), r[None, :, :512],
                         r[None, :, 512:], np.arange(n)[None], np.array([n])))
    wkv = mi.f64(wl.wkv_b)
    keys = 0
    passes = 0
    t0 = time.perf_counter()
    while passes < repeats or time.perf_counter() - t0 < min_seconds:
        for qn, qp, c, pe, idx, ep in prepared:
            orc.decode_absorbed(qn, qp, wkv, c, pe, idx, ep, wl.scale)
            keys += idx.shape[1]
        passes += 1
    dt = time.perf_counter() - t0
    return keys * HEADS / dt, dt, threads, passes


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import torch

    import mla_inputs as mi
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    wl = mi.make_config(args.config, device=dev,
                        batch=slice(0, min(8, mi.CONFIG_SPECS[args.config]["B"])))
    rows = list(range(wl.B))
    for _ in range(args.warmup):
        oracle_sample_rate(wl, rows[:1])
    rates, secs, threads = [], 0.0, 1
    for _ in range(args.steps):
        r, dt, threads, _ = oracle_sample_rate(wl, rows)
        rates.append(r)
        secs += dt
    value = len(rates) * len(rows) * wl.k * HEADS / secs
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args.config, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{len(rows)} batch rows of the workload per step "
                                   f"(selected rows only), float64 numpy oracle"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(cid: int, world: int):
    desc = {
        0: ("tiny dense decode B=1 end_pos=1001 all 1001 selected", 1, 1001),
        1: ("decode B=8 end_pos=4096 top-k=2048", 8, 2048),
        2: ("decode B=64 end_pos=32768 top-k=2048", 64, 2048),
        3: ("decode B=128 end_pos~U[4096,131072] top-k=2048 (1024 recent + 1024 older), "
            "bf16 cache [128,131072,576]", 128, 2048),
        4: ("cache-write B=32 at 65535 + decode top-k=2048 over 65536", 32, 2048),
    }[cid]
    return {"workload": desc[0], "batch_per_gpu": desc[1], "global_batch": desc[1] * world,
            "top_k": desc[2], "heads": HEADS, "latent": 512, "rope": 64,
            "l2": "flushed between steps (256 MiB write, then a 256 MiB read of a second buffer so "
                  "that the flush's own dirty lines are written back before the timed step)",
            "parallelism": f"replicas x{world}"}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def time_next_rows(B, dev, stream, flush_l2, n_op, world, peaks):
    """Times the two rows after the decode on the attention block's path at
    batch B: the output projection and the query path, each call after an L2
    flush, CUDA events on the launching stream, max over ranks."""
    import torch

    import mla_inputs as mi
    import sparse_head_latent_absorbed_b200 as shla

    next_rows = {}
    o_in, w_o = mi.make_out_proj(B=B, seed=1, device=dev)
    d_out = torch.empty(B, 7168, dtype=torch.bfloat16, device=dev)
    op_ws = torch.empty(shla.mla_out_proj_workspace_bytes(B), dtype=torch.uint8, device=dev)
    for _ in range(3):
        shla.mla_out_proj(o_in, w_o, out=d_out, ws=op_ws)
    torch.cuda.synchronize()
    op_ms = 0.0
    for _ in range(n_op):
        flush_l2()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        shla.mla_out_proj(o_in, w_o, out=d_out, ws=op_ws)
        b_.record(stream)
        torch.cuda.synchronize()
        op_ms += a.elapsed_time(b_)
    op_ms = reduce_max(op_ms / n_op, world, dev)
    op_bytes = 7168 * 16384 * 2 + B * 16384 * 2 + B * 7168 * 2
    next_rows["out_proj"] = {
        "what": "Delta = flatten(O) W_O^T, W_O [7168, 16384] bf16 (xwt_kernel + xwt_finish_bf16)",
        "us": op_ms * 1e3, "bound": "hbm", "algorithmic_bytes": op_bytes,
        "achieved": op_bytes / (op_ms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
        "frac": op_bytes / (op_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    del w_o
    qx, wq_a, qn_w, wq_b, qrope, qpos = mi.make_query_proj(B=B, seed=1, device=dev)
    q_ws = torch.empty(shla.mla_query_proj_workspace_bytes(B), dtype=torch.uint8, device=dev)
    for _ in range(3):
        shla.mla_query_proj(qx, wq_a, qn_w, 1e-6, wq_b, qrope, qpos, ws=q_ws)
    torch.cuda.synchronize()
    q_ms = 0.0
    for _ in range(n_op):
        flush_l2()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        shla.mla_query_proj(qx, wq_a, qn_w, 1e-6, wq_b, qrope, qpos, ws=q_ws)
        b_.record(stream)
        torch.cuda.synchronize()
        q_ms += a.elapsed_time(b_)
    q_ms = reduce_max(q_ms / n_op, world, dev)
    q_bytes = (1536 * 7168 + 24576 * 1536) * 2 + B * 7168 * 2 + B * 128 * 192 * 2
    next_rows["query_proj"] = {
        "what": "x -> wq_a -> RMSNorm -> wq_b -> split -> RoPE (2 x xwt_kernel + finishes)",
        "us": q_ms * 1e3, "bound": "hbm", "algorithmic_bytes": q_bytes,
        "achieved": q_bytes / (q_ms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
        "frac": q_bytes / (q_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    del wq_a, wq_b
    return next_rows


def time_multi_query_rows(wl, dev, stream, flush_l2, n_op, world, peaks):
    """Times the rows built on mla_decode_mq, each call after an L2 flush:
    sparse prefill of one 4096-token prompt (top-k 2048, causal) and, when a
    decode workload `wl` is given, multi-query decode of two new tokens per
    sequence on its cache.  Work counts only listed positions inside each
    query row's causal limit."""
    import torch

    import mla_inputs as mi
    import sparse_head_latent_absorbed_b200 as shla

    def timed(w):
        ws = torch.empty(shla.mla_decode_workspace_bytes(w.B, w.k), dtype=torch.uint8,
                         device=dev)
        out = torch.empty(w.B, HEADS, 128, dtype=torch.bfloat16, device=dev)

        def call():
            shla.mla_decode_mq(w.q_nope, w.q_pe, w.wkv_b, w.cache, w.topk, w.end_pos, w.scale,
                               w.queries_per_row, out=out, ws=ws)
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        ms = 0.0
        for _ in range(n_op):
            flush_l2()
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            call()
            b_.record(stream)
            torch.cuda.synchronize()
            ms += a.elapsed_time(b_)
        ms = reduce_max(ms / n_op, world, dev)
        valid = int(((w.topk >= 0) & (w.topk < w.end_pos[:, None])).sum().item())
        return ms, valid

    rows = {}
    pf = mi.make_prefill(B=1, S=4096, k=2048, seed=1, device=dev)
    ms, valid = timed(pf)
    # absorbed form (what runs): 2 x 128 x (576 + 512) flop per listed key, plus
    # the fold and W_UV of each query row; the pages' form of the prefill
    # branch: 2 x 128 x (192 + 128) flop per listed key, plus expanding each
    # prompt position's keys and values for the 128 heads (2 x 128 x 512 x 256)
    absorbed = valid * 278_528 + pf.B * 33_554_432
    pages = valid * 81_920 + pf.B * 33_554_432
    rows["prefill"] = {
        "what": "sparse prefill, 1 prompt x 4096 tokens, top-k 2048, causal (mla_decode_mq, "
                "query row = token, absorbed form); the 4.7 MB prompt cache stays in L2",
        "us": ms * 1e3, "headline": "head_keys_per_s",
        "head_keys_per_s": valid * HEADS / (ms * 1e-3), "listed_keys": valid,
        "absorbed_form_flops": absorbed, "pages_form_flops": pages,
        "absorbed_tflops": absorbed / (ms * 1e-3) / 1e12,
        "absorbed_frac_of_bf16_peak": absorbed / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
        "note": "the fraction is tensor-pipe occupancy by the absorbed form, not speed on "
                "the pages' form of the work; the headline is head*keys/s"}
    del pf
    if wl is not None:
        mq = mi.make_multi_query(B=wl.B, S=2, T=wl.T, k=wl.k, seed=1, device=dev,
                                 cache=wl.cache, end_pos=wl.end_pos, wkv_b=wl.wkv_b)
        ms, valid = timed(mq)
        nbytes = valid * 1156 + mq.B * (32768 + 16384 + 32768) + 33_554_432
        rows["multi_query_decode"] = {
            "what": f"multi-query decode, {wl.B} sequences x 2 new tokens, top-k {wl.k}, on the "
                    "decode workload's cache (mla_decode_mq)",
            "us": ms * 1e3, "head_keys_per_s": valid * HEADS / (ms * 1e-3),
            "listed_keys": valid, "bound": "hbm", "algorithmic_bytes": nbytes,
            "achieved": nbytes / (ms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    return rows


def run_next_rows_only(args, dev, world, rank):
    """Times only the next rows (output projection, query path) at the
    workload's batch, with no decode cache on the device: the small case
    under which those kernels are profiled.  Prints one JSON line."""
    import torch

    import mla_inputs as mi
    B = mi.CONFIG_SPECS[args.config]["B"]
    flush_w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def flush_l2():
        flush_w.zero_()
        flush_r.max()
    n_op = max(3, min(args.steps, 100))
    peaks = load_peaks()
    rows = time_next_rows(B, dev, torch.cuda.current_stream(), flush_l2, n_op, world, peaks)
    rows.update(time_multi_query_rows(None, dev, torch.cuda.current_stream(), flush_l2, n_op,
                                      world, peaks))
    if rank == 0:
        print(json.dumps({"next_rows": rows, "batch": B, "n_gpus": world,
                          "l2": "flushed before each call"}), flush=True)
    return 0


def run_ours(args):
    import torch

    rank, world, local = dist_env()
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    import mla_inputs as mi
    import sparse_head_latent_absorbed_b200 as shla

    if args.only_next_rows:
        return run_next_rows_only(args, dev, world, rank)
    wl = mi.make_config(args.config, device=dev)
    B, k = wl.B, wl.k
    ws = torch.empty(shla.mla_decode_workspace_bytes(B, k), dtype=torch.uint8, device=dev)
    out = torch.empty(B, HEADS, 128, dtype=torch.bfloat16, device=dev)
    status = torch.zeros(2, dtype=torch.int32, device=dev)
    flush_w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def flush_l2():
        # writing 256 MiB evicts L2 but leaves it full of dirty lines; reading
        # another 256 MiB writes those back here rather than in the timed step
        flush_w.zero_()
        flush_r.max()
    stream = torch.cuda.current_stream()
    write = args.config == 4
    cw_ws = None
    if write:
        cw_ws = torch.empty(shla.mla_cache_write_workspace_bytes(B), dtype=torch.uint8, device=dev)
        tab = wl.rope[wl.write_pos:wl.write_pos + 1].contiguous()

    def step():
        if write:
            shla.mla_cache_write(wl.x, wl.w_kva, wl.norm_w, wl.eps, tab, wl.write_pos, wl.cache,
                                 ws=cw_ws)
        shla.mla_decode(wl.q_nope, wl.q_pe, wl.wkv_b, wl.cache, wl.topk, wl.end_pos, wl.scale,
                        out=out, ws=ws, status=status)

    # fold, attend, W_UV; the combine kernel runs when rows are split
    launches_per_step = 3 + (1 if shla.mla_decode_num_splits(B, k) > 1 else 0) \
        + (2 if write else 0)

    # ---- device-timed steps ----
    # The clock sampler runs from the timed steps through the phase and
    # end-to-end loops below, so that its record covers far more than the
    # timed region alone (a few ms at the default step count).
    clk = ClockSampler(dev).__enter__()
    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()
    clk.wait_live()
    barrier(world)
    clk_start = clk.mark()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for i in range(args.steps):
        flush_l2()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk_timed_end = clk.mark()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = reduce_max(sum(step_ms), world, dev)
    ms_per_step = total_ms / args.steps
    if int(status[0]) != 0:
        raise RuntimeError(f"kernel status word reports a timeout: {status.tolist()}")

    # ---- the attend kernel alone (roofline of the dominant kernel) ----
    phase_ms = {1: [], 2: [], 3: []}
    if not write:
        n_rep = max(3, min(args.steps, 200))
        for i in range(n_rep + 3):
            flush_l2()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            ev[0].record(stream)
            for ph in (1, 2, 3):
                shla.mla_decode_phase(ph, wl.q_nope, wl.q_pe, wl.wkv_b, wl.cache, wl.topk,
                                      wl.end_pos, wl.scale, out, ws, status)
                ev[ph].record(stream)
            torch.cuda.synchronize()
            if i >= 3:
                for ph in (1, 2, 3):
                    phase_ms[ph].append(ev[ph - 1].elapsed_time(ev[ph]))
    peaks = load_peaks()
    cache_write = None
    if write:
        # the cache write alone (kv = x W_KVa, RMSNorm, RoPE, row store), each
        # call after an L2 flush: bound by streaming W_KVa once
        n_rep = max(3, min(args.steps, 200))
        cw_ms = []
        for i in range(n_rep + 3):
            flush_l2()
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            shla.mla_cache_write(wl.x, wl.w_kva, wl.norm_w, wl.eps, tab, wl.write_pos, wl.cache,
                                 ws=cw_ws)
            b_.record(stream)
            torch.cuda.synchronize()
            if i >= 3:
                cw_ms.append(a.elapsed_time(b_))
        cw = reduce_max(statistics.mean(cw_ms), world, dev)
        cw_bytes = 7168 * 576 * 2 + B * (7168 * 2 + 576 * 2)
        cache_write = {"what": "cache write of B rows: kv = x W_KVa (split-K tcgen05) + RMSNorm + "
                               "RoPE + bf16 store (cw_gemm_kernel + cw_finalize_kernel)",
                       "us": cw * 1e3, "bound": "hbm", "algorithmic_bytes": cw_bytes,
                       "achieved": cw_bytes / (cw * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                       "unit": "GB/s",
                       "frac": cw_bytes / (cw * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    roofline = None
    if phase_ms[2]:
        core_ms = reduce_max(statistics.mean(phase_ms[2]), world, dev)
        cb, cf = core_kernel_work(B, k)
        achieved = cb / (core_ms * 1e-3) / 1e9
        roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": achieved / peaks["hbm_gbs"], "traffic": profiled_traffic(),
                    "kernel": "core_kernel (gather + QK^T + softmax + PV)",
                    "kernel_us": core_ms * 1e3,
                    "tensor_tflops": cf / (core_ms * 1e-3) / 1e12,
                    "tensor_frac_of_bf16_peak": cf / (core_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                    "peak_source": peaks["source"] + " (burst copy)",
                    "step_frac": algorithmic_work(B, k)[0] / (ms_per_step * 1e-3) / 1e9
                    / peaks["hbm_gbs"],
                    "step_frac_what": "the whole step's algorithmic bytes / its time / peak",
                    "phase_us": {"fold": 1e3 * statistics.mean(phase_ms[1]),
                                 "attend": 1e3 * statistics.mean(phase_ms[2]),
                                 "merge_uv": 1e3 * statistics.mean(phase_ms[3])}}

    # ---- end to end through the public API with host buffers ----
    h_qn = wl.q_nope.cpu().pin_memory()
    h_qp = wl.q_pe.cpu().pin_memory()
    h_ix = wl.topk.cpu().pin_memory()
    h_ep = wl.end_pos.cpu().pin_memory()
    h_out = torch.empty(B, HEADS, 128, dtype=torch.bfloat16).pin_memory()
    d_qn, d_qp = torch.empty_like(wl.q_nope), torch.empty_like(wl.q_pe)
    d_ix, d_ep = torch.empty_like(wl.topk), torch.empty_like(wl.end_pos)
    h2d = sum(t.numel() * t.element_size() for t in (h_qn, h_qp, h_ix, h_ep))
    d2h = h_out.numel() * h_out.element_size()

    def e2e_step():
        d_qn.copy_(h_qn, non_blocking=True)
        d_qp.copy_(h_qp, non_blocking=True)
        d_ix.copy_(h_ix, non_blocking=True)
        d_ep.copy_(h_ep, non_blocking=True)
        if write:
            shla.mla_cache_write(wl.x, wl.w_kva, wl.norm_w, wl.eps, tab, wl.write_pos, wl.cache,
                                 ws=cw_ws)
        shla.mla_decode(d_qn, d_qp, wl.wkv_b, wl.cache, d_ix, d_ep, wl.scale, out=out, ws=ws)
        h_out.copy_(out, non_blocking=True)

    n_e2e = max(3, min(args.steps, 200))
    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e_ms = 0.0
    for _ in range(n_e2e):
        flush_l2()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e2e_step()
        b_.record(stream)
        torch.cuda.synchronize()
        e_ms += a.elapsed_time(b_)
    e_ms = reduce_max(e_ms / n_e2e, world, dev)
    clk.__exit__(None, None, None)
    clocks = clk.summary(clk_start)
    clocks["timed_region_samples"] = clk_timed_end - clk_start
    clocks["covers"] = "timed steps, per-phase timing loop and end-to-end loop"

    # ---- the next rows on the path: output projection and query path ----
    next_rows = {}
    if not args.no_next_rows:
        n_op = max(3, min(args.steps, 100))
        next_rows = time_next_rows(B, dev, stream, flush_l2, n_op, world, peaks)
        next_rows.update(time_multi_query_rows(wl, dev, stream, flush_l2, n_op, world, peaks))

    units = B * k * HEADS
    value = world * units / (ms_per_step * 1e-3)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "us_per_step": ms_per_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded, distributions of the workload; no public dataset involved)",
        "config": workload_config(args.config, world),
        "roofline": roofline,
        **({"cache_write": cache_write} if cache_write else {}),
        "e2e": {"value": world * units / (e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
                "what": "H2D of q_nope, q_pe, top-k, end_pos from pinned host memory, "
                        "mla_decode, D2H of O; cache and weights resident"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "algorithmic": dict(zip(("bytes_per_step", "flops_per_step"), algorithmic_work(B, k))),
        "next_rows": next_rows,
    }
    # ---- CPU baseline: the oracle on a bounded sample, rank 0 at N=1 ----
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        rows = list(range(min(args.cpu_rows, B)))
        rate, dt, threads, passes = oracle_sample_rate(wl, rows, min_seconds=args.cpu_seconds)
        line["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": f"{len(rows)} of {B} batch rows (their selected rows "
                                          f"only), {passes} passes, {dt:.1f} s"}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=3, choices=[0, 1, 2, 3, 4])
    ap.add_argument("--cpu-rows", type=int, default=128)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="minimum seconds of oracle work in the cpu_baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip the separate timing of the output projection and query path")
    ap.add_argument("--only-next-rows", action="store_true",
                    help="time only the output projection and query path (no decode cache "
                         "on the device; prints their next_rows object)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
