"""Benchmark: one MLA decode step (append -> absorb -> decode + combine -> output_up) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Prints ONE JSON line (rank 0).  A step is one pass of the whole hot path over one batch:
the workload's new tokens are appended to the paged latent cache, their queries absorbed,
attention runs over the cache (split-KV + combine) and W_UV is applied.  Inputs are seeded
synthetic data resident in HBM before timing starts; the cache read per step (hundreds of
MB) is larger than the 126 MB L2, so no separate flush is done.  Multi-GPU runs are
independent replicas (one per rank, no data-path collective), timed as the max over ranks.

--impl reference times the fp64 CPU oracle on the host cores on a bounded sample of the same
workload (the reference arm; there is no other implementation to run).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import pathlib
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MLA decode TFLOP/s & HBM GB/s vs roofline (H=128,B=64,L=8192)"
DEFAULT_WORKLOAD = "v3_bf16"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- algorithmic units

def step_units(w, lengths):
    """Algorithmic FLOPs and HBM bytes of one step, per step row, from the workload sizes.

    Attention: 2(d_c + d_rope) + 2 d_c FLOPs per (query token, head, attended token); bytes =
    cache bytes of the attended tokens + packed Q + o_lat.  Projections: 2*m*n*k FLOPs and
    their weight + activation bytes."""
    import numpy as np
    lengths = np.asarray(lengths, dtype=np.int64)
    s_q, H = w.s_q, w.n_heads
    T = len(lengths) * s_q
    act_b = 4 if w.act_dtype == "f32" else 2
    tok_b = {"f32": 4 * w.row_width, "bf16": 2 * w.row_width, "fp8": w.d_c + 4 * (w.d_c // 128) + 2 * w.d_rope}[w.cache_dtype]
    if w.causal or s_q > 1:
        attended = sum(int(L - s_q + j + 1) for L in lengths for j in range(s_q) if L - s_q + j + 1 > 0)
    else:
        attended = int(lengths.sum()) * s_q
    per_pair = 2 * (w.d_c + w.d_rope) + 2 * w.d_c
    u = {}
    u["decode_flops"] = per_pair * H * attended
    u["decode_bytes"] = int(lengths.sum()) * tok_b + T * H * w.row_width * act_b + T * H * w.d_c * act_b
    u["append_flops"] = 2 * T * w.d_model * w.row_width
    u["append_bytes"] = (w.row_width * w.d_model + T * w.d_model) * act_b + T * tok_b
    u["absorb_flops"] = 2 * T * H * w.d_nope * w.d_c
    u["absorb_bytes"] = (H * w.d_nope * w.d_c + T * H * (w.d_nope + w.d_rope) + T * H * w.row_width) * act_b
    u["output_flops"] = 2 * T * H * w.d_c * w.d_v
    u["output_bytes"] = (H * w.d_v * w.d_c + T * H * w.d_c + T * H * w.d_v) * act_b
    u["step_flops"] = u["decode_flops"] + u["append_flops"] + u["absorb_flops"] + u["output_flops"]
    u["step_bytes"] = u["decode_bytes"] + u["append_bytes"] + u["absorb_bytes"] + u["output_bytes"]
    u["attended"] = attended
    return u


# ----------------------------------------------------------------------------- clocks (NVML, read only)

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read-only queries) every ~20 ms."""

    REASONS = {  # bit -> name (nvmlClocksEventReason*)
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        try:
            from mla_latent_kv_27_b200.runner import nvml_handle
            self.nv, self.h = nvml_handle(device_index)
            pynvml = self.nv
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report it instead of clocks
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, reasons))
            except Exception:
                pass
            time.sleep(0.02)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0, t1):
        if not self.ok:
            return {"error": getattr(self, "err", "nvml unavailable")}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        src = inside or self.samples[-3:]
        if not src:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = statistics.median(s[1] for s in src)
        bits = 0
        for s in src:
            bits |= s[2]
        names = sorted(n for b, n in self.REASONS.items() if bits & b and n != "gpu_idle")
        return {"sm_mhz": mhz, "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(inside), "window_s": round(t1 - t0, 3)}


# ----------------------------------------------------------------------------- our arm

def workload_from_args(args):
    """The named workload, optionally resized (--batch / --length) for profiling runs."""
    import dataclasses

    from mla_latent_kv_27_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    if args.batch or args.length:
        batch = args.batch or w.batch
        length = args.length or int(wl.draw_lengths(w).max())
        w = dataclasses.replace(w, name=f"{w.name}[B={batch},L={length}]", batch=batch,
                                lengths=(length,) * batch, len_range=None)
    return w


# ----------------------------------------------------------------------------- ranks
# One process per GPU, each a full replica of the workload; the only collectives are a barrier
# around the timed regions and the max over ranks of each rank's device time.  Every rank takes
# the same collective steps in the same order.

def rank_barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (the slowest rank sets the job's
    time); the identity without a multi-rank process group.  `device` is where the reduction
    tensor lives: a CUDA device under NCCL, the CPU under gloo."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1):
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def whole_job_rate(units_per_rank, world, ms):
    """Units per second of the whole job: every rank processed `units_per_rank` in at most
    `ms` milliseconds (weak scaling: the per-rank work is fixed as the rank count grows)."""
    return units_per_rank * world / (ms * 1e-3)


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch

    import mla_latent_kv_27_b200 as mla
    from mla_latent_kv_27_b200 import workloads as wl
    from mla_latent_kv_27_b200.runner import MLARunner

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workload_from_args(args)
    runner = MLARunner(w, device=dev, n_split=args.n_split)
    if w.cache_dtype == "fp8":
        runner.fill_cache_projected()
    else:
        runner.fill_cache_direct()
    runner.draw_step_inputs()
    torch.cuda.synchronize()
    units = step_units(w, runner.lengths)
    stream = torch.cuda.current_stream()

    barrier = rank_barrier

    # warm-up
    for _ in range(args.warmup):
        runner.step()
    torch.cuda.synchronize()
    st, detail = mla.mla_check_device_error()
    if st != 0:
        raise RuntimeError(f"device error word after warm-up: status {st} detail {detail:#x}")

    # timed region: K steps, events around the whole region only (an event recorded between two
    # kernels ends the programmatic dependent launch overlap of the second), then K decode calls
    # each bracketed by events on the same stream for the roofline of the dominant kernel
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dec = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.1)
    barrier()
    torch.cuda.synchronize()
    launches0 = mla.mla_launch_count()
    t0 = time.perf_counter()
    ev0.record(stream)
    for i in range(args.steps):
        runner.step()
    ev1.record(stream)
    torch.cuda.synchronize()
    launches = mla.mla_launch_count() - launches0
    for i in range(args.steps):
        dec[i][0].record(stream)
        runner.decode()
        dec[i][1].record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    barrier()
    sampler.stop()
    ms_total = ev0.elapsed_time(ev1)
    dec_ms = [a.elapsed_time(b) for a, b in dec]
    dec_avg = sum(dec_ms) / len(dec_ms)
    ms_total, dec_avg = max_over_ranks([ms_total, dec_avg], dev)
    ms_step = ms_total / args.steps

    # end to end through the public API with host buffers: every step copies its inputs from
    # pinned host memory and its output back, on copy streams that overlap the previous and
    # next steps' kernels (MLARunner.run_host_steps)
    from mla_latent_kv_27_b200.runner import bind_host_to_device
    import os
    cpus_before = os.sched_getaffinity(0)
    local_cpus = bind_host_to_device(dev)  # pinned buffers on the GPU's NUMA node
    h_in = [runner.h_new.cpu().pin_memory(), runner.q_nope.cpu().pin_memory(), runner.q_rope.cpu().pin_memory()]
    out_host = torch.empty(runner.out.shape, dtype=runner.out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in h_in)
    d2h = out_host.numel() * out_host.element_size()
    e2e_steps = max(1, min(args.steps, 200))

    def host_steps(k):
        runner.run_host_steps([h_in[0]] * k, [h_in[1]] * k, [h_in[2]] * k, [out_host] * k)

    host_steps(3)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    host_steps(e2e_steps)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    # the same transfers alone (H2D on one stream, D2H on another): the end-to-end step cannot be
    # shorter than this, whatever the kernels do, and it varies with the host link of the box
    s_in, s_out = runner._copy_streams
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    for _ in range(e2e_steps):
        with torch.cuda.stream(s_in):
            runner.h_new.copy_(h_in[0], non_blocking=True)
            runner.q_nope.copy_(h_in[1], non_blocking=True)
            runner.q_rope.copy_(h_in[2], non_blocking=True)
        with torch.cuda.stream(s_out):
            out_host.copy_(runner.out, non_blocking=True)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    c1.record(stream)
    torch.cuda.synchronize()
    copy_ms = c0.elapsed_time(c1) / e2e_steps
    os.sched_setaffinity(0, cpus_before)
    e2e_ms, copy_ms = max_over_ranks([e2e_ms, copy_ms], dev)
    barrier()

    if rank != 0:
        return None
    peaks, peaks_src = load_peaks()
    hbm_peak = peaks["hbm_gbs"]
    tflops_step = whole_job_rate(units["step_flops"], world, ms_step) / 1e12
    dec_gbs = units["decode_bytes"] / (dec_avg * 1e-3) / 1e9
    dec_tflops = units["decode_flops"] / (dec_avg * 1e-3) / 1e12
    ridge = peaks["bf16_tflops"] * 1e3 / hbm_peak  # FLOP per byte
    intensity = units["decode_flops"] / units["decode_bytes"]
    bound = "hbm" if intensity < ridge else "tensor"
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": round(dec_gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(dec_gbs / hbm_peak, 4)}
    else:
        roof = {"bound": "tensor", "achieved": round(dec_tflops, 1), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(dec_tflops / peaks["bf16_tflops"], 4)}
    roof_time_us = max(units["decode_bytes"] / (hbm_peak * 1e9), units["decode_flops"] / (peaks["bf16_tflops"] * 1e12)) * 1e6
    roof.update({
        "traffic": measured_traffic(w), "kernel": "mla_decode_attention (decode + split combine)",
        "peak_source": peaks_src, "flops_per_launch": units["decode_flops"],
        "bytes_per_launch": units["decode_bytes"], "avg_launch_us": round(dec_avg * 1e3, 2),
        "roofline_us": round(roof_time_us, 2), "frac_of_roofline_time": round(roof_time_us / (dec_avg * 1e3), 4),
        "decode_tflops": round(dec_tflops, 1), "decode_gbs": round(dec_gbs, 1),
    })
    clocks = sampler.summary(t0, t1)
    line = {
        "metric": METRIC, "value": round(tflops_step, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.act_dtype if w.cache_dtype != "fp8" else "bf16+fp8cache",
        "data": "synthetic (seeded; cache rows drawn N(0,1) as W_DKV h produces; fp8 cache built by the append kernel)",
        "config": workload_config(w, runner.lengths, runner.n_split, world),
        "hbm_gbs": round(whole_job_rate(units["step_bytes"], world, ms_step) / 1e9, 1),
        "roofline": roof,
        "e2e": {"value": round(whole_job_rate(units["step_flops"], world, e2e_ms) / 1e12, 3), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 5), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "host_cpus_local_to_gpu": len(local_cpus) if local_cpus else None,
                "copies_alone_ms_per_step": round(copy_ms, 5)},
        "gpu_launches": int(launches), "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_seconds)
    return line


# ----------------------------------------------------------------------------- the oracle on the host

def _oracle_sample(w, lengths, seed=0):
    """Seeded numpy inputs for the oracle's step on the given sequences (drawn like the
    GPU arm's inputs, not copied from the device)."""
    import numpy as np
    from mla_latent_kv_27_b200 import workloads as wl
    r = np.random.default_rng([w.seed, 77, seed])
    B = len(lengths)
    T = B * w.s_q
    w_dkv, w_kr, w_uk, w_uv = (x.astype(np.float64) for x in wl.draw_weights(w))
    total = int(sum(lengths))
    rows = r.standard_normal((total, w.row_width))
    table, n_pages = wl.make_block_table(lengths, 0, False, None)
    pages = wl.scatter_rows_to_pages(rows, lengths, table, n_pages)
    h_new = r.standard_normal((T, w.d_model))
    q_nope = r.standard_normal((T, w.n_heads, w.d_nope))
    q_rope = r.standard_normal((T, w.n_heads, w.d_rope))
    pos = (np.repeat(lengths, w.s_q) - w.s_q + np.tile(np.arange(w.s_q), B)).astype(np.int64)
    return dict(w_dkv=w_dkv, w_kr=w_kr, w_uk=w_uk, w_uv=w_uv, pages=pages, table=table, h_new=h_new,
                q_nope=q_nope, q_rope=q_rope, pos=pos, lengths=np.asarray(lengths))


def _oracle_step(w, s):
    from oracle import mla_oracle as orc
    orc.compress_kv(s["h_new"], s["w_dkv"], s["w_kr"], s["pos"], w.theta)
    q_lat, q_rot = orc.absorb_query(s["q_nope"], s["q_rope"], s["pos"], s["w_uk"], w.theta)
    o, _ = orc.decode_paged(q_lat, q_rot, s["pages"], s["table"], s["lengths"], w.s_q, w.scale, w.d_c, 64,
                            causal=w.causal or w.s_q > 1)
    return orc.output_up(o, s["w_uv"])


def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(w, budget_s=12.0, n_seq=None):
    """Time the fp64 oracle's step on a bounded sample: the first n_seq sequences of the
    workload (all of its step rows: append of their new tokens, absorb, decode, output_up),
    repeated until about budget_s seconds have passed."""
    from mla_latent_kv_27_b200 import workloads as wl
    lengths = wl.draw_lengths(w)
    if n_seq is None:
        n_seq = max(1, min(len(lengths), 4))
    sample_lengths = lengths[:n_seq]
    s = _oracle_sample(w, sample_lengths)
    units = step_units(w, sample_lengths)
    reps, t0 = 0, time.perf_counter()
    while True:
        _oracle_step(w, s)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or reps >= 1000:
            break
    v = units["step_flops"] * reps / el / 1e12
    return {"value": round(v, 6), "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
            "sample": f"{n_seq} of {len(lengths)} sequences of {w.name} (lengths {list(map(int, sample_lengths))}), "
                      f"full step rows, {reps} repetitions in {el:.1f} s, numpy fp64"}


# DRAM traffic of one decode call (decode kernel + combine), read from the ncu summaries under
# profiles/: a summary records it on a line
#   traffic-record: <workload> <bytes per call> <hash of the decode sources it was captured on>
# (dram__bytes_read.sum + dram__bytes_write.sum of the call's kernels in one capture of the bench's
# own workload).  A workload without a record, or whose record was taken on other kernel sources,
# reports null.
TRAFFIC_SOURCES = ("decode_tc.cu", "decode_sh.cu", "decode_plan.cuh", "decode_tc.cuh", "sm100_ptx.cuh",
                   "mla_internal.cuh")


def kernel_source_hash():
    """Hash of the decode sources' code: comments and blank lines are left out, so that editing a
    comment does not orphan a traffic record."""
    import hashlib
    import re
    h = hashlib.sha256()
    csrc = pathlib.Path(__file__).resolve().parent / "mla_latent_kv_27_b200" / "csrc"
    for name in TRAFFIC_SOURCES:
        code = re.sub(r"//[^\n]*", "", (csrc / name).read_text())
        h.update("\n".join(line.rstrip() for line in code.splitlines() if line.strip()).encode())
    return h.hexdigest()[:16]


def traffic_records():
    import re
    recs = {}
    prof = pathlib.Path(__file__).resolve().parent / "profiles"
    for md in sorted(prof.glob("*.md")):
        for m in re.finditer(r"^traffic-record: (\S+) (\d+) ([0-9a-f]{16})\s*$", md.read_text(), re.M):
            recs.setdefault(m.group(1), []).append((int(m.group(2)), m.group(3)))
    return recs


def measured_traffic(w):
    """The recorded bytes when this is the stock workload and the same kernel sources."""
    from mla_latent_kv_27_b200 import workloads as wl
    if w != wl.WORKLOADS.get(w.name):
        return None
    h = kernel_source_hash()
    for nbytes, src in traffic_records().get(w.name, []):
        if src == h:
            return nbytes
    return None


def workload_config(w, lengths, n_split, world):
    return {"workload": w.name, "batch": len(lengths), "heads": w.n_heads, "s_q": w.s_q,
            "d_model": w.d_model, "d_c": w.d_c, "d_rope": w.d_rope,
            "lengths": {"min": int(lengths.min()), "max": int(lengths.max()), "sum": int(lengths.sum())},
            "cache_dtype": w.cache_dtype, "n_split": n_split,
            "partition": "length-balanced over 74 SM pairs (the tensor-core path ignores n_split)",
            "l2": "inputs larger than L2 (cache read per step > 126 MB); no flush",
            "parallelism": f"replicas x{world}"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    from mla_latent_kv_27_b200 import workloads as wl
    w = workload_from_args(args)
    lengths = wl.draw_lengths(w)
    n_seq = max(1, min(len(lengths), 2))
    s = _oracle_sample(w, lengths[:n_seq])
    units = step_units(w, lengths[:n_seq])
    for _ in range(args.warmup):
        _oracle_step(w, s)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(w, s)
    el = time.perf_counter() - t0
    ms = el * 1e3 / args.steps
    v = units["step_flops"] / (ms * 1e-3) / 1e12
    sample = f"{n_seq} of {len(lengths)} sequences of {w.name} per step, full step rows, numpy fp64"
    return {
        "metric": METRIC, "value": round(v, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)", "impl": "reference",
        "config": dict(workload_config(w, lengths, w.n_split if args.n_split is None else args.n_split, world),
                       sample=sample),
        "cpu_baseline": {"value": round(v, 6), "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(v, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=0, help="resize the workload (profiling runs)")
    ap.add_argument("--length", type=int, default=0, help="fixed length for every sequence (profiling runs)")
    ap.add_argument("--n-split", type=int, default=None, help="KV chunks per sequence (default: workload's)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
