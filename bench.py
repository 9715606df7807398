"""Benchmark of the multi-pattern dilated-attention forward on B200.

One step = one forward over the whole workload (all patterns, segment split,
dilated gather, attention, scatter and combination: a single launch of the
library) on inputs already resident in HBM.  Default workload: 32K tokens,
5 patterns (the pages' experiment pattern set), bf16, causal.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--impl ours|reference] [--sweep]

With N > 1 (launched under torch.distributed.run) every rank runs its own
independent copy of the workload (different seed): the path has no data
exchange, so this is weak scaling with no collective on the data path.

Prints one JSON line (rank 0).  Timing: CUDA events on the launch stream per
step, with a 512 MiB L2 flush between steps (outside the events), barrier +
synchronize around the timed region, max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Dilated-attn fwd tokens/s @32K, 5 patterns; % of bf16 tensor-core peak"
UNIT = "tokens/s"
METRIC_BWD = "Dilated-attn bwd (dq, dk, dv) tokens/s; % of the kernel's roofline peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_BF16_TFLOPS = 2250.0
# fp32 FMA peak: 148 SMs x 128 FP32 lanes x 2 flops x 1.965 GHz (clocks.max.sm)
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# The sources a kernel family's device code is built from: its own file and
# the shared headers (code only: comments and layout are ignored).  A change
# anywhere else leaves its counters valid.
_FAMILY_SOURCES = ("device_util.cuh", "params.h", "tc_ptx.cuh")


def _code_only(text: str) -> str:
    """C/C++ source without comments and with whitespace collapsed: the part
    a comment or layout edit does not change."""
    import re

    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash(family: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_long_sequence_attn_b200", "csrc")
    src = {"patterns": "perpattern.cu"}.get(family, f"{family}.cu")
    paths = [os.path.join(csrc, n) for n in (src,) + _FAMILY_SOURCES]
    paths.append(os.path.join(ROOT, "include", "longnet.h"))
    for path in paths:
        with open(path, encoding="utf-8") as f:
            h.update(os.path.basename(path).encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def traffic_from_profiles(workload: str, impl_name: str):
    """DRAM bytes per launch from a committed ncu summary, when it was taken
    on the current kernel sources; None otherwise."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    ent = d.get(f"{impl_name}:{workload}")
    if not ent or ent.get("source_hash") != kernel_source_hash(impl_name):
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while running
    (read-only; no setting of the GPU is touched)."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml

            pynvml.nvmlInit()
            import torch

            uuid = None
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            except Exception:
                uuid = None
            if uuid:
                u = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
                self.h = pynvml.nvmlDeviceGetHandleByUUID(u.encode() if isinstance(u, str) else u)
            else:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.err = repr(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                t = time.time()
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                reasons = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((t, mhz, reasons))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.th = threading.Thread(target=self._run, daemon=True)
            self.th.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.th.join()

    def summary(self, t0: float, t1: float):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        note = None
        if not inside:
            inside = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:3]
            note = "timed region shorter than the sampling period; nearest samples"
        reasons = set()
        for _, _, bits in inside:
            for bit, name in self.REASONS.items():
                if bits & bit and name != "gpu_idle":
                    reasons.add(name)
        out = {"sm_mhz": statistics.median([s[1] for s in inside]) if inside else None,
               "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons), "samples": len(inside)}
        if note:
            out["note"] = note
        return out


def dist_env():
    from sparse_long_sequence_attn_b200.replicas import dist_env as _de

    return _de()


_INPUT_CACHE = {}


def oracle_cpu_sample(wl, n_positions: int, seed: int):
    """Time the fp64 oracle (as it stands) on n_positions random positions of
    the workload, all heads of each position.  Returns (tokens/s, seconds,
    threads, description)."""
    import numpy as np

    import oracle
    from sparse_long_sequence_attn_b200 import workloads as wlm

    key = (wl.name, wl.N)
    if key not in _INPUT_CACHE:
        _INPUT_CACHE.clear()
        _INPUT_CACHE[key] = wlm.make_inputs(wl)
    q, k, v = _INPUT_CACHE[key]
    g = np.random.default_rng(seed)
    pos = g.choice(wl.N, size=n_positions, replace=False)
    bs = g.integers(0, wl.B, size=n_positions)
    rows = np.array([(b, p, h) for b, p in zip(bs, pos) for h in range(wl.H)], dtype=np.int64)
    t0 = time.perf_counter()
    oracle.dilated_attn_rows_fp64(q, k, v, wl.patterns, rows, wl.causal)
    dt = time.perf_counter() - t0
    desc = (f"{n_positions} random positions (all {wl.H} heads each) of workload {wl.name}, "
            f"fp64 oracle rows entry point")
    return n_positions / dt, dt, oracle.num_threads(), desc


def run_reference(args, wl):
    """Reference arm: the fp64 CPU oracle timed on the host cores, on a
    bounded sample of the same workload per step."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import numpy as np  # noqa: F401

    n_pos = args.ref_positions
    times = []
    threads = None
    desc = None
    for i in range(args.warmup + args.steps):
        tps, dt, threads, desc = oracle_cpu_sample(wl, n_pos, seed=1000 + i)
        if i >= args.warmup:
            times.append(dt)
    mean_dt = sum(times) / len(times)
    value = n_pos / mean_dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean_dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "N": wl.N, "H": wl.H, "D": wl.D,
                   "patterns": [list(p) for p in wl.patterns], "causal": wl.causal,
                   "sample_positions_per_step": n_pos},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long32k")
    ap.add_argument("--impl", default="ours", help="ours | reference")
    ap.add_argument("--kernel", default="auto",
                    help="auto | simt | tcgen05 | smallseg | patterns (forward); auto | simt | tiles | tcgen05 (--pass bwd)")
    ap.add_argument("--ref-positions", type=int, default=48)
    ap.add_argument("--cpu-positions", type=int, default=0,
                    help="oracle sample size for cpu_baseline (0: calibrate to ~10 s)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true", help="linear-scaling sweep instead")
    ap.add_argument("--no-sweep", action="store_true",
                    help="leave the linear-scaling sweep out of the default line")
    ap.add_argument("--no-variants", action="store_true",
                    help="leave the one-change variants of the 32K shape out of the default line")
    ap.add_argument("--soak-s", type=float, default=1.0,
                    help="seconds of repeated steps after the timed region, for the clock record")
    ap.add_argument("--pass", dest="pass_", default="fwd", choices=("fwd", "bwd"),
                    help="fwd: the forward (default); bwd: the backward (dq, dk, dv)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    from sparse_long_sequence_attn_b200 import workloads as wlm

    if args.workload.startswith("sweep") and args.workload[5:].isdigit():
        wl = wlm.sweep_workload(int(args.workload[5:]))  # one sweep size, e.g. sweep65536
    else:
        wl = wlm.WORKLOADS[args.workload]
    if args.impl == "reference":
        if args.pass_ == "bwd":
            return run_reference_bwd(args, wl)
        return run_reference(args, wl)
    if args.sweep:
        return run_sweep(args)
    if args.pass_ == "bwd":
        return run_backward(args, wl)
    return run_ours(args, wl)


def _impl_code(name):
    from sparse_long_sequence_attn_b200 import binding as bd

    return {"auto": bd.LONGNET_IMPL_AUTO, "simt": bd.LONGNET_IMPL_SIMT,
            "tcgen05": bd.LONGNET_IMPL_TCGEN05, "smallseg": bd.LONGNET_IMPL_SMALLSEG,
            "patterns": bd.LONGNET_IMPL_PATTERNS}[name]


def _impl_name(code):
    return {1: "simt", 2: "tcgen05", 3: "smallseg", 5: "patterns"}.get(code, str(code))


def time_steps(fn, steps, warmup, stream, flush_buf):
    """Warm up, then time each step with CUDA events on `stream`, flushing L2
    between steps outside the events.  Returns per-step seconds."""
    import torch

    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for i in range(steps):
        with torch.cuda.stream(stream):
            flush_buf.zero_()
            evs[i][0].record(stream)
            fn()
            evs[i][1].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) * 1e-3 for a, b in evs]


def run_ours(args, wl):
    import torch
    import torch.distributed as dist

    from sparse_long_sequence_attn_b200 import binding as bd
    from sparse_long_sequence_attn_b200 import workloads as wlm

    ws, rank, local = dist_env()
    if ws > 1:
        torch.cuda.set_device(local)
        # a short timeout: a rank left waiting for a dead peer ends with an error
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if ws > 1 else 0)
    torch.cuda.set_device(dev)
    bd.load_library()

    from sparse_long_sequence_attn_b200.replicas import max_over_ranks, replica_seed, weak_scaling_rate

    q, k, v = wlm.make_inputs(wl, seed=replica_seed(wl.seed, rank))
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    out = torch.empty_like(qd)
    lse = torch.empty((wl.B, wl.H, wl.N), device=dev, dtype=torch.float32)
    impl = _impl_code(args.kernel)
    chosen = bd.longnet_select_impl(wl.B, wl.N, wl.H, wl.D, wl.patterns, wl.causal, wl.torch_dtype) \
        if impl == bd.LONGNET_IMPL_AUTO else impl
    stream = torch.cuda.Stream(device=dev)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def step():
        bd.longnet_dilated_attn_fwd(qd, kd, vd, out, lse, wl.patterns, wl.causal, impl, stream)

    # device-resident timed region
    sampler = ClockSampler(dev.index)
    sampler.start()
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    per_step = time_steps(step, args.steps, args.warmup, stream, flush)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall1 = time.time()
    sampler.stop()
    st = bd.longnet_last_device_status(stream)
    if st != 0:
        raise RuntimeError(f"device status after the timed region: {bd.status_string(st)}")
    total = max_over_ranks(sum(per_step), dev)
    mean_step = total / args.steps

    # clock soak (after the timed region, not part of `value`): the same step
    # repeated for at least a second, with the clocks sampled throughout, so
    # the clock record is a distribution even when the timed region is short
    soak = None
    if args.soak_s > 0:
        soak_sampler = ClockSampler(dev.index)
        soak_sampler.start()
        torch.cuda.synchronize()
        s0 = time.time()
        n_soak, soak_dev_s = 0, 0.0
        while time.time() - s0 < args.soak_s:
            per = time_steps(step, 50, 0, stream, flush)
            n_soak += len(per)
            soak_dev_s += sum(per)
        s1 = time.time()
        soak_sampler.stop()
        soak = {"steps": n_soak, "ms_per_step": soak_dev_s / n_soak * 1e3,
                "clocks": soak_sampler.summary(s0, s1)}

    # end-to-end through the public API with host buffers: pinned H2D of the
    # inputs, the forward, D2H of out and lse, every step: the C-ABI call on
    # host buffers (longnet_dilated_attn_fwd_host), whose head chunks overlap
    # their copies with the attention
    out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    lse_h = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)

    def e2e_step():
        bd.longnet_dilated_attn_fwd_host(qh, kh, vh, out_h, lse_h, qd, kd, vd, out, lse, wl.patterns, wl.causal,
                                         impl, stream)

    e2e_steps = max(3, min(args.steps, 20))
    if ws > 1:
        dist.barrier()
    per_e2e = time_steps(e2e_step, e2e_steps, 2, stream, flush)
    e2e_total = max_over_ranks(sum(per_e2e), dev)
    h2d = sum(x.numel() * x.element_size() for x in (qh, kh, vh))
    d2h = out_h.numel() * out_h.element_size() + lse_h.numel() * lse_h.element_size()

    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    tokens = wl.B * wl.N
    value = weak_scaling_rate(tokens, ws, mean_step)
    flops = wlm.algorithmic_flops(wl)
    peaks, peak_kind = load_peaks()
    kname = _impl_name(chosen)
    if kname == "smallseg":
        achieved = wlm.algorithmic_bytes(wl) / mean_step / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"]}
    else:
        achieved = flops / mean_step / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"]}
    roof["peak_source"] = f"{peak_kind} ({'MEASURED_PEAKS.json' if peak_kind == 'measured' else 'recipe fallback'})"
    roof["traffic"] = traffic_from_profiles(wl.name, kname)
    roof["algorithmic_flops_per_launch"] = flops
    # secondary: the exact causal pair count (4*D flops per pair) instead of
    # the nominal w/r formula
    pairs = wlm.exact_pair_count(wl)
    roof["exact_pairs_per_launch"] = pairs
    roof["tflops_exact_pairs"] = 4.0 * wl.D * pairs / mean_step / 1e12
    roof["algorithmic_bytes_per_launch"] = wlm.algorithmic_bytes(wl)
    roof["frac_of_sustained_bf16"] = flops / mean_step / 1e12 / peaks.get("bf16_tflops_sustained", 1400.0)
    roof["frac_of_nominal_bf16"] = flops / mean_step / 1e12 / NOMINAL_BF16_TFLOPS

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": mean_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": {"bf16": "bf16", "fp16": "f16", "fp32": "f32"}[wl.dtype],
        "data": "synthetic: seeded N(0,1) q/k/v at the workload's shape (no dataset)",
        "config": {"workload": wl.name, "B": wl.B, "N": wl.N, "H": wl.H, "D": wl.D,
                   "patterns": [list(p) for p in wl.patterns], "causal": wl.causal,
                   "global_batch": wl.B * ws, "seq_len": wl.N,
                   "parallelism": f"independent replicas x{ws}" if ws > 1 else "single GPU",
                   "kernel": kname, "l2": "512 MiB flush between timed steps (outside events)"},
        "roofline": roof,
        "e2e": {"value": weak_scaling_rate(tokens * e2e_steps, ws, e2e_total), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "call": "longnet_dilated_attn_fwd_host (pinned host buffers; pieces of batches, heads or "
                        "positions overlap their copies with the attention)"},
        "gpu_launches": (1 + len(wl.patterns) if kname == "patterns" else 1) * args.steps,
        "clocks": sampler.summary(t_wall0, t_wall1),
    }
    if soak is not None:
        line["clock_soak"] = soak
    if ws == 1 and wl.name == "long32k" and not args.no_sweep:
        line["sweep"] = sweep_lines(args.steps, args.warmup, args.kernel, dev.index)
        line["sweep_linear_1M_vs_64K"] = line["sweep"][-1]["tokens_per_s_vs_65536"]
    if ws == 1 and wl.name == "long32k" and not args.no_variants:
        line["variants"] = variant_lines(args.steps, args.warmup, dev.index)
        line["backward"] = backward_line(wl, args.steps, args.warmup, dev.index)
    if ws == 1 and not args.no_cpu_baseline:
        n = args.cpu_positions
        calibrate = n <= 0
        if calibrate:
            tps, dt, _, _ = oracle_cpu_sample(wl, 16, seed=1)
            n = int(max(16, min(wl.N, 10.0 * tps)))
        tps, dt, threads, desc = oracle_cpu_sample(wl, n, seed=2)
        if calibrate and dt < 5.0 and n < wl.N:
            # a small probe understates the threads' throughput: size again
            n = int(min(wl.N, n * 10.0 / max(dt, 1e-3)))
            tps, dt, threads, desc = oracle_cpu_sample(wl, n, seed=3)
        line["cpu_baseline"] = {"value": tps, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": desc + f" ({dt:.1f} s)"}
    print(json.dumps(line), flush=True)
    return 0


def oracle_bwd_sample(wl, n_positions: int, seed: int):
    """Time the fp64 oracle's per-row backward (as it stands) on n_positions
    random positions, all heads each.  Returns (tokens/s, seconds, threads,
    description)."""
    import numpy as np

    import oracle
    from sparse_long_sequence_attn_b200 import workloads as wlm

    key = ("bwd", wl.name, wl.N)
    if key not in _INPUT_CACHE:
        _INPUT_CACHE.clear()
        q, k, v = wlm.make_inputs(wl)
        _INPUT_CACHE[key] = (q, k, v, wlm.random_cotangent(wl.B, wl.N, wl.H, wl.D,
                                                           wl.torch_dtype, seed=wl.seed))
    q, k, v, dout = _INPUT_CACHE[key]
    g = np.random.default_rng(seed)
    pos = g.choice(wl.N, size=n_positions, replace=False)
    bs = g.integers(0, wl.B, size=n_positions)
    rows = np.array([(b, p, h) for b, p in zip(bs, pos) for h in range(wl.H)], dtype=np.int64)
    t0 = time.perf_counter()
    oracle.dilated_attn_bwd_rows_fp64(q, k, v, dout, wl.patterns, rows, wl.causal)
    dt = time.perf_counter() - t0
    desc = (f"{n_positions} random positions (all {wl.H} heads each) of workload {wl.name}, "
            f"fp64 oracle per-row backward (dq, dk, dv of each row)")
    return n_positions / dt, dt, oracle.num_threads(), desc


def run_reference_bwd(args, wl):
    """Reference arm of the backward: the fp64 oracle's per-row backward on a
    bounded sample of positions per step, on the host cores."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    n_pos = max(1, args.ref_positions // 16)
    times, threads, desc = [], None, None
    for i in range(args.warmup + args.steps):
        _, dt, threads, desc = oracle_bwd_sample(wl, n_pos, seed=1000 + i)
        if i >= args.warmup:
            times.append(dt)
    mean_dt = sum(times) / len(times)
    value = n_pos / mean_dt
    line = {
        "impl": "reference", "metric": METRIC_BWD, "value": value, "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean_dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": wl.name, "pass": "bwd", "B": wl.B, "N": wl.N, "H": wl.H,
                   "D": wl.D, "patterns": [list(p) for p in wl.patterns], "causal": wl.causal,
                   "sample_positions_per_step": n_pos},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_backward(args, wl):
    """The backward (dq, dk, dv) of the workload: the CUDA forward runs once
    before timing to give out and lse; a step is one longnet_dilated_attn_bwd
    call (two kernels)."""
    import torch
    import torch.distributed as dist

    from sparse_long_sequence_attn_b200 import binding as bd
    from sparse_long_sequence_attn_b200 import workloads as wlm
    from sparse_long_sequence_attn_b200.replicas import max_over_ranks, replica_seed, weak_scaling_rate

    ws, rank, local = dist_env()
    if ws > 1:
        torch.cuda.set_device(local)
        # a short timeout: a rank left waiting for a dead peer ends with an error
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if ws > 1 else 0)
    torch.cuda.set_device(dev)
    bd.load_library()
    seed = replica_seed(wl.seed, rank)
    q, k, v = wlm.make_inputs(wl, seed=seed)
    dout = wlm.random_cotangent(wl.B, wl.N, wl.H, wl.D, wl.torch_dtype, seed=seed)
    qd, kd, vd, dod = (x.to(dev) for x in (q, k, v, dout))
    out, lse = bd.dilated_attn(qd, kd, vd, wl.patterns, wl.causal)
    dq, dk, dv = (torch.empty(qd.shape, dtype=torch.float32, device=dev) for _ in range(3))
    impl = {"auto": bd.LONGNET_IMPL_AUTO, "simt": bd.LONGNET_IMPL_SIMT, "tiles": bd.LONGNET_IMPL_TILES,
            "tcgen05": bd.LONGNET_IMPL_TCGEN05}[args.kernel]
    # the family AUTO runs: the first of tcgen05, tiles that takes the call
    # (one untimed probe call each), else SIMT
    family = {bd.LONGNET_IMPL_SIMT: "simt", bd.LONGNET_IMPL_TILES: "tiles",
              bd.LONGNET_IMPL_TCGEN05: "tcgen05"}.get(impl)
    if family is None:
        family = "simt"
        for name, code in (("tcgen05", bd.LONGNET_IMPL_TCGEN05), ("tiles", bd.LONGNET_IMPL_TILES)):
            try:
                bd.longnet_dilated_attn_bwd(qd, kd, vd, out, lse, dod, dq, dk, dv, wl.patterns, wl.causal, code)
                family = name
                break
            except bd.LongNetError as e:
                if e.code != bd.LONGNET_ERR_UNSUPPORTED:
                    raise
    tiles = family in ("tiles", "tcgen05")  # tensor cores
    stream = torch.cuda.Stream(device=dev)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    torch.cuda.synchronize()

    def step():
        bd.longnet_dilated_attn_bwd(qd, kd, vd, out, lse, dod, dq, dk, dv, wl.patterns, wl.causal,
                                    impl, stream)

    sampler = ClockSampler(dev.index)
    sampler.start()
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    per_step = time_steps(step, args.steps, args.warmup, stream, flush)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall1 = time.time()
    sampler.stop()
    st = bd.longnet_last_device_status(stream)
    if st != 0:
        raise RuntimeError(f"device status after the timed region: {bd.status_string(st)}")
    mean_step = max_over_ranks(sum(per_step), dev) / args.steps

    # end to end: pinned H2D of q, k, v, out, lse, dout; the backward; D2H of
    # dq, dk, dv
    hosts = [x.cpu().pin_memory() for x in (qd, kd, vd, out, lse, dod)]
    devs = (qd, kd, vd, out, lse, dod)
    grads_h = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in (dq, dk, dv)]

    def e2e_step():
        with torch.cuda.stream(stream):
            for d_, h_ in zip(devs, hosts):
                d_.copy_(h_, non_blocking=True)
            bd.longnet_dilated_attn_bwd(qd, kd, vd, out, lse, dod, dq, dk, dv, wl.patterns,
                                        wl.causal, impl, stream)
            for h_, d_ in zip(grads_h, (dq, dk, dv)):
                h_.copy_(d_, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 10))
    if ws > 1:
        dist.barrier()
    per_e2e = time_steps(e2e_step, e2e_steps, 2, stream, flush)
    e2e_total = max_over_ranks(sum(per_e2e), dev)
    h2d = sum(x.numel() * x.element_size() for x in hosts)
    d2h = sum(x.numel() * x.element_size() for x in grads_h)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    tokens = wl.B * wl.N
    pairs = wlm.exact_pair_count(wl)
    # 10*D flops per pair: the score and dP products and the dq, dk, dv sums
    # (the tile kernels execute 14*D: S and dP are computed in both kernels)
    flops = 10.0 * wl.D * pairs
    achieved = flops / mean_step / 1e12
    peaks, peak_kind = load_peaks()
    if tiles:
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                "peak_source": f"{peak_kind} bf16 GEMM "
                               f"({'MEASURED_PEAKS.json' if peak_kind == 'measured' else 'recipe fallback'})",
                "traffic": traffic_from_profiles(wl.name + ":bwd", "backward" if family == "tiles"
                                                 else "bwd_tcgen05"),
                "kernel": ("bwd_dkv_tile_kernel + bwd_dq_tile_kernel (one call)" if family == "tiles" else
                           "bwd_delta_kernel + bwd_tc_kernel keys (dk, dv) + bwd_tc_kernel queries (dq)"),
                "executed_flops_per_launch": 14.0 * wl.D * pairs}
    else:
        roof = {"bound": "alu", "achieved": achieved, "peak": FP32_ALU_TFLOPS, "unit": "TFLOP/s",
                "frac": achieved / FP32_ALU_TFLOPS,
                "peak_source": "derived: 148 SMs x 128 fp32 FMA lanes x 2 x 1.965 GHz",
                "traffic": None, "kernel": "bwd_dkv_kernel + bwd_dq_kernel (one call)"}
    roof["exact_pairs_per_launch"] = pairs
    roof["algorithmic_flops_per_launch"] = flops
    line = {
        "metric": METRIC_BWD, "value": weak_scaling_rate(tokens, ws, mean_step), "unit": UNIT,
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": mean_step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": (f"{wl.dtype} (fp32 accumulate, fp32 gradients)" if tiles else "f32"),
        "data": "synthetic: seeded N(0,1) q/k/v/dout at the workload's shape (no dataset)",
        "config": {"workload": wl.name, "pass": "bwd", "B": wl.B, "N": wl.N, "H": wl.H,
                   "D": wl.D, "patterns": [list(p) for p in wl.patterns], "causal": wl.causal,
                   "global_batch": wl.B * ws, "seq_len": wl.N,
                   "parallelism": f"independent replicas x{ws}" if ws > 1 else "single GPU",
                   "kernel": {"tiles": "tiles (mma.sync)", "tcgen05": "tcgen05 (TMA, TMEM)"}.get(family, "simt"),
                   "l2": "512 MiB flush between timed steps (outside events)"},
        "roofline": roof,
        "e2e": {"value": weak_scaling_rate(tokens * e2e_steps, ws, e2e_total), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": (3 if family == "tcgen05" else 2) * args.steps,
        "clocks": sampler.summary(t_wall0, t_wall1),
    }
    if ws == 1 and not args.no_cpu_baseline:
        tps, dt, _, _ = oracle_bwd_sample(wl, 1, seed=1)
        n = int(max(1, min(wl.N, 10.0 * tps)))
        tps, dt, threads, desc = oracle_bwd_sample(wl, n, seed=2)
        line["cpu_baseline"] = {"value": tps, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": desc + f" ({dt:.1f} s)"}
    print(json.dumps(line), flush=True)
    return 0


def sweep_lines(steps, warmup, kernel="auto", dev_index=0):
    """Linear-scaling sweep: the forward at N = 65536, 262144, 1048576 (B 1,
    H 8, six patterns of sparse length 2048), each timed over `steps` steps
    with CUDA events and an L2 flush between steps.  Inputs are drawn on the
    device (the sweep measures speed; its parity is tested separately)."""
    import torch

    from sparse_long_sequence_attn_b200 import binding as bd
    from sparse_long_sequence_attn_b200 import workloads as wlm

    dev = torch.device("cuda", dev_index)
    stream = torch.cuda.Stream(device=dev)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    impl = _impl_code(kernel)
    peaks, _ = load_peaks()
    res = []
    for N in wlm.SWEEP_NS:
        wl = wlm.sweep_workload(N)
        g = torch.Generator(device=dev)
        g.manual_seed(wl.seed)
        qd, kd, vd = (torch.randn(wl.B, N, wl.H, wl.D, device=dev, generator=g,
                                  dtype=torch.float32).to(torch.bfloat16) for _ in range(3))
        out = torch.empty_like(qd)
        lse = torch.empty((wl.B, wl.H, N), device=dev, dtype=torch.float32)

        def step():
            bd.longnet_dilated_attn_fwd(qd, kd, vd, out, lse, wl.patterns, wl.causal, impl, stream)

        per = time_steps(step, steps, warmup, stream, flush)
        st = bd.longnet_last_device_status(stream)
        if st != 0:
            raise RuntimeError(f"device status after the sweep at N={N}: {bd.status_string(st)}")
        t = sum(per) / len(per)
        tf = wlm.algorithmic_flops(wl) / t / 1e12
        res.append({"N": N, "ms": t * 1e3, "tokens_per_s": N / t, "tflops": tf,
                    "frac": tf / peaks["bf16_tflops"]})
        del qd, kd, vd, out, lse
        torch.cuda.empty_cache()
    base = res[0]["tokens_per_s"]
    for r in res:
        r["tokens_per_s_vs_65536"] = r["tokens_per_s"] / base
    return res


def backward_line(wl, steps, warmup, dev_index=0):
    """The backward (dq, dk, dv) of the same workload after its forward, timed
    like the main line: ms per call, the family AUTO ran, and the algorithmic
    rate (10 D flops per attended pair) against the bf16 peak."""
    import torch

    from sparse_long_sequence_attn_b200 import binding as bd
    from sparse_long_sequence_attn_b200 import workloads as wlm

    dev = torch.device("cuda", dev_index)
    stream = torch.cuda.Stream(device=dev)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    q, k, v = (x.to(dev) for x in wlm.make_inputs(wl))
    dout = wlm.random_cotangent(wl.B, wl.N, wl.H, wl.D, wl.torch_dtype, seed=wl.seed).to(dev)
    out, lse = bd.dilated_attn(q, k, v, wl.patterns, wl.causal)
    dq, dk, dv = (torch.empty(q.shape, dtype=torch.float32, device=dev) for _ in range(3))
    family = "tiles or simt"
    try:
        bd.longnet_dilated_attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, wl.patterns, wl.causal,
                                    bd.LONGNET_IMPL_TCGEN05)
        family = "tcgen05"
    except bd.LongNetError as e:
        if e.code != bd.LONGNET_ERR_UNSUPPORTED:
            raise

    def step():
        bd.longnet_dilated_attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, wl.patterns, wl.causal,
                                    bd.LONGNET_IMPL_AUTO, stream)

    per = time_steps(step, steps, warmup, stream, flush)
    st = bd.longnet_last_device_status(stream)
    if st != 0:
        raise RuntimeError(f"device status after the backward: {bd.status_string(st)}")
    t = sum(per) / len(per)
    flops = 10.0 * wl.D * wlm.exact_pair_count(wl)
    peaks, peak_kind = load_peaks()
    tf = flops / t / 1e12
    res = {"ms": t * 1e3, "steps": steps, "family": family, "tokens_per_s": wl.B * wl.N / t,
           "tflops_algorithmic": tf, "frac_of_bf16_peak": tf / peaks["bf16_tflops"], "peak_source": peak_kind}
    del q, k, v, dout, out, lse, dq, dk, dv
    torch.cuda.empty_cache()
    # the same shape at D = 128 (half the heads, the same FLOPs)
    H2, D2 = wl.H // 2, 2 * wl.D
    g = torch.Generator(device=dev)
    g.manual_seed(wl.seed)
    q, k, v, dout = (torch.randn(wl.B, wl.N, H2, D2, device=dev, generator=g, dtype=torch.float32)
                     .to(wl.torch_dtype) for _ in range(4))
    out, lse = bd.dilated_attn(q, k, v, wl.patterns, wl.causal)
    dq, dk, dv = (torch.empty(q.shape, dtype=torch.float32, device=dev) for _ in range(3))
    per = time_steps(lambda: bd.longnet_dilated_attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, wl.patterns,
                                                         wl.causal, bd.LONGNET_IMPL_AUTO, stream),
                     steps, warmup, stream, flush)
    st = bd.longnet_last_device_status(stream)
    if st != 0:
        raise RuntimeError(f"device status after the D = 128 backward: {bd.status_string(st)}")
    t2 = sum(per) / len(per)
    res["d128"] = {"H": H2, "D": D2, "ms": t2 * 1e3, "tflops_algorithmic": flops / t2 / 1e12,
                   "frac_of_bf16_peak": flops / t2 / 1e12 / peaks["bf16_tflops"]}
    del q, k, v, dout, out, lse, dq, dk, dv
    torch.cuda.empty_cache()
    return res


def variant_lines(steps, warmup, dev_index=0):
    """The 32K-token shape (B 1, H 12, D 64, five patterns, causal) with one
    thing changed at a time, each timed like the main line (CUDA events, L2
    flush between steps): the input options through the prologue pass
    (longnet_dilated_attn_fwd_ws: qk_norm, XPOS), qk_norm inside the kernel
    (longnet_dilated_attn_fwd_ex, which AUTO sends to the family that takes
    it), a sequence 64 tokens short (a partial last segment), D = 128
    (H 6) and D = 32 (H 24).  Reports the family AUTO picked for each.  Inputs drawn on the
    device; parity of each variant is tested separately."""
    import torch

    from sparse_long_sequence_attn_b200 import binding as bd
    from sparse_long_sequence_attn_b200 import workloads as wlm

    dev = torch.device("cuda", dev_index)
    stream = torch.cuda.Stream(device=dev)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    base = wlm.WORKLOADS["long32k"]
    res = []
    cases = [("plain", base.N, base.H, base.D, "plain"), ("qk_norm_prologue", base.N, base.H, base.D, "ws_norm"),
             ("xpos_prologue", base.N, base.H, base.D, "ws_xpos"),
             ("qk_norm_in_kernel", base.N, base.H, base.D, "ex_norm"),
             ("qk_norm_in_kernel_d128", base.N, base.H // 2, 128, "ex_norm"),
             ("partial_last_segment", base.N - 64, base.H, base.D, "plain"),
             ("d128", base.N, base.H // 2, 128, "plain"), ("d32", base.N, base.H * 2, 32, "plain")]
    for name, N, H, D, mode in cases:
        g = torch.Generator(device=dev)
        g.manual_seed(base.seed)
        qd, kd, vd = (torch.randn(base.B, N, H, D, device=dev, generator=g,
                                  dtype=torch.float32).to(torch.bfloat16) for _ in range(3))
        out = torch.empty_like(qd)
        lse = torch.empty((base.B, H, N), device=dev, dtype=torch.float32)
        qk_norm = mode in ("ws_norm", "ex_norm")
        xpos = mode == "ws_xpos"
        ws = None
        if mode.startswith("ws"):
            ws = torch.empty(bd.longnet_fwd_workspace_bytes(base.B, N, H, D, torch.bfloat16, qk_norm, xpos),
                             dtype=torch.uint8, device=dev)

        def step():
            if ws is not None:
                bd.longnet_dilated_attn_fwd_ws(qd, kd, vd, out, lse, base.patterns, base.causal, ws,
                                               bd.LONGNET_IMPL_AUTO, stream, qk_norm, xpos)
            else:
                bd.longnet_dilated_attn_fwd(qd, kd, vd, out, lse, base.patterns, base.causal,
                                            bd.LONGNET_IMPL_AUTO, stream, qk_norm)

        # one untimed call to see how long a step takes; slow families get fewer steps
        t0 = time.time()
        step()
        torch.cuda.synchronize()
        n = steps if time.time() - t0 < 0.05 else 3
        per = time_steps(step, n, min(warmup, 3), stream, flush)
        st = bd.longnet_last_device_status(stream)
        if st != 0:
            raise RuntimeError(f"device status after variant {name}: {bd.status_string(st)}")
        fam = _impl_name(bd.longnet_select_impl(base.B, N, H, D, base.patterns, base.causal, torch.bfloat16))
        t = sum(per) / len(per)
        res.append({"variant": name, "N": N, "H": H, "D": D, "family": fam, "steps": n,
                    "ms": t * 1e3, "tokens_per_s": base.B * N / t})
        del qd, kd, vd, out, lse, ws
        torch.cuda.empty_cache()
    return res


def run_sweep(args):
    """Linear-scaling sweep alone: one JSON line {"sweep": [...]}."""
    import torch

    torch.cuda.set_device(0)
    from sparse_long_sequence_attn_b200 import binding as bd

    bd.load_library()
    print(json.dumps({"sweep": sweep_lines(args.steps, args.warmup, args.kernel)}), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
