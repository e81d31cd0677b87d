#!/usr/bin/env python
"""Benchmark of the exact-attention hot path: one step = forward + backward
(fa_forward, then the three backward stages that fa_backward runs) over one batch
of seeded synthetic inputs already resident in HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the fp64 CPU oracle on the host cores

Metric: attention fwd+bwd TFLOP/s, counting 4*B*H*N^2*d for the forward (halved
when causal) and 2.5x that for the backward. Timing: CUDA events on the launching
stream around every kernel of every step; L2 is flushed (a 256 MiB write) before
each timed step, and the step's launches are queued ahead (a short GPU-side spin),
both outside the events; W untimed warm-up steps; a barrier and a
device synchronise on both sides of the K timed steps; max over ranks. With N > 1
each rank runs its own replica of the workload (independent heads; no collective
on the data path), so the scaling is weak. nvidia-smi samples the clocks during
the timed region; a hardware or thermal slowdown, or SM clocks held far below
their maximum with no reason active, takes the measurement again, once.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd/bwd TFLOP/s (bf16, d=128) and % of B200 dense BF16 peak"
DEFAULT_WORKLOAD = "long_b1h8_n16384_d128"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
L2_FLUSH_BYTES = 256 << 20
# A GPU-side spin of this many clocks (about 100 us) before each timed region, outside its
# events: the host has then queued every launch of the region before the GPU reaches the
# first event, so the events time the kernels and not the Python call overhead between them.
QUEUE_AHEAD_CYCLES = 200_000


def parse():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--seq-len", type=int, default=None,
                    help="override the workload's N (same B, H, d, dtype, mask and scale)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the secondary configurations (rank 0, one GPU only)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle sample")
    ap.add_argument("--reference-seconds", type=float, default=150.0,
                    help="--impl reference: CPU time of the whole run (warm-up and timed "
                         "steps), split evenly over the steps")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_sha():
    """Hash of the CUDA sources; ncu traffic figures are only reported while the
    kernels are the ones they were taken on."""
    csrc = os.path.join(ROOT, "io_aware_attention_flashattention_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        table = json.load(f)
    ent = table.get(kernel)
    if not ent or ent.get("workload") != workload or ent.get("source_sha") != kernel_source_sha():
        return None
    return ent.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(self.index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        return summarise_clock_lines(self.lines)


def summarise_clock_lines(lines):
    """Median SM clock, the highest max clock and power, and the throttle reasons seen
    active, from `nvidia-smi --format=csv,noheader,nounits` lines of the fields in
    ClockSampler.FIELDS. Lines that do not parse (a header, a cut-off last line) are
    skipped."""
    sm, smax, power, reasons = [], [], [], set()
    for line in lines:
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            smax.append(float(parts[2]))
            power.append(float(parts[3]))
        except ValueError:
            continue
        for name, val in zip(ClockSampler.NAMES, parts[5:9]):
            if val.lower() == "active":
                reasons.add(name)
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": max(smax) if smax else None,
            "power_w_max": max(power) if power else None,
            "reasons": sorted(reasons), "samples": len(sm)}


REJECTING_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")
PINNED_LOW_FRACTION = 0.75


def clock_verdict(clocks):
    """Why a timed region's clock record rejects its number, or None if it stands.

    A hardware or thermal slowdown rejects it. So does a median SM clock below
    PINNED_LOW_FRACTION of the maximum with no reason active (a clock lock left behind
    by someone else). sw_power_cap alone is normal under a dense load and is kept. No
    samples (no nvidia-smi) gives no verdict."""
    bad = [r for r in clocks.get("reasons", []) if r in REJECTING_REASONS]
    if bad:
        return "throttled: " + ",".join(bad)
    sm, smax = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    if sm is not None and smax and not clocks.get("reasons") and sm < PINNED_LOW_FRACTION * smax:
        return f"SM clock {sm:.0f} MHz of {smax:.0f} MHz with no reason active"
    return None


# ---------------------------------------------------------------- ranks


def replica_seed(w, rank: int) -> int:
    """Each rank draws its own replica of the workload (independent heads)."""
    return w.seed + 7919 * rank


def max_over_ranks(value_ms: float, world: int, device=None) -> float:
    """The slowest rank's time (the job's time); a no-op for one rank. Uses the
    default process group (NCCL on GPUs; gloo works for host-side tests)."""
    if world <= 1:
        return float(value_ms)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def workload_config(w, world: int) -> dict:
    """The ``config`` object of the JSON line; both arms print the same one."""
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
            "scale": w.scale, "parallelism": f"replicas{world}",
            "l2": "flushed (256 MiB write) before every timed step"}


def visible_pairs(N: int, causal: bool, window=None, block_mask=None) -> int:
    """Number of (query, key) pairs the masks keep, for one head: causal keeps j <= i,
    a window (left, right) keeps i - left <= j <= i + right (negative = unbounded), a
    block mask over 128 x 128 blocks keeps (i, j) iff mask[i // 128][j // 128]."""
    import numpy as np

    i = np.arange(N, dtype=np.int64)
    lo = np.zeros(N, dtype=np.int64)
    hi = np.full(N, N - 1, dtype=np.int64)
    if causal:
        hi = np.minimum(hi, i)
    if window is not None:
        left, right = window
        if left >= 0:
            lo = np.maximum(lo, i - left)
        if right >= 0:
            hi = np.minimum(hi, i + right)
    if block_mask is None:
        return int(np.maximum(hi - lo + 1, 0).sum())
    m = np.asarray(block_mask) != 0
    T = m.shape[0]
    total = 0
    for kb in range(T):  # keys of block kb visible to each row: [max(lo, kb*128), min(hi, ...)]
        k0, k1 = kb * 128, min(N, kb * 128 + 128) - 1
        cnt = np.maximum(np.minimum(hi, k1) - np.maximum(lo, k0) + 1, 0)
        total += int((cnt * m[i // 128, kb]).sum())
    return total


def job_throughput(flops_per_step: float, world: int, steps: int, job_ms: float) -> float:
    """Whole-job TFLOP/s: the work of all ranks divided by the slowest rank's time."""
    return flops_per_step * world * steps / (job_ms * 1e-3) / 1e12


# ---------------------------------------------------------------- CPU oracle sample


def oracle_sample(w, seconds: float, rng_seed: int = 0, inputs=None):
    """The fp64 oracle, as it stands, on a bounded sample of the workload: R random
    (head, query row) pairs through the forward (O, LSE) and the dQ backward rows,
    each with all visible keys. Returns (flops, seconds, rows, threads). Flops count
    what the oracle's definition computes per visible (row, key) pair and head
    dimension element: 4 for the forward (S and PV), 6 for the dQ rows (S, dP and
    dS K)."""
    import numpy as np

    import oracle
    from io_aware_attention_flashattention_b200.inputs import workload_inputs

    q, k, v, do = inputs if inputs is not None else workload_inputs(w)
    # fp64 copies made once, outside the timed calls
    q, k, v, do = (np.ascontiguousarray(t.double().numpy()) for t in (q, k, v, do))
    BH = w.B * w.H
    rng = np.random.default_rng(rng_seed)

    def run(R):
        heads = rng.integers(0, BH, R)
        rows = rng.integers(0, w.N, R)
        order = np.lexsort((rows, heads))
        heads, rows = heads[order], rows[order]
        t0 = time.perf_counter()
        oracle.forward_rows(q, k, v, w.scale, w.causal, heads, rows)
        oracle.backward_dq_rows(q, k, v, do, w.scale, w.causal, heads, rows)
        dt = time.perf_counter() - t0
        visible = (rows + 1) if w.causal else np.full(R, w.N)
        return float(np.sum(visible)) * w.d * 10.0, dt

    r0 = max(32, 4 * oracle.num_threads())
    run(r0)  # warm-up: thread pool start-up and cold caches, not timed
    _, t0 = run(r0)  # calibration: enough rows to occupy every thread
    per_row = t0 / r0
    R = int(max(1, seconds / max(per_row, 1e-9)))
    flops, dt = run(R)
    if dt < 0.6 * seconds:  # calibration overestimated the row cost: top up once
        R2 = int(max(1, (seconds - dt) * R / max(dt, 1e-9)))
        f2, dt2 = run(R2)
        flops, dt, R = flops + f2, dt + dt2, R + R2
    return flops, dt, R, oracle.num_threads()


def oracle_one_thread(seconds: float = 1.5) -> dict:
    """The oracle on one host thread, on the two small workloads (the fp32 oracle-scale
    one and the GPT-2 shape): TFLOP/s of a bounded row sample each, for comparison with
    the all-core figure."""
    import oracle
    from io_aware_attention_flashattention_b200.inputs import WORKLOADS

    n = oracle.num_threads()
    out = {}
    try:
        oracle.default().set_num_threads(1)
        for name in ("oracle_f32_n256_d64", "gpt2_causal_b8h12_n1024_d64"):
            f, t, R, _ = oracle_sample(WORKLOADS[name], seconds, rng_seed=7)
            out[name] = {"value": f / t / 1e12, "rows": R, "seconds": round(t, 2)}
    finally:
        oracle.default().set_num_threads(n)
    return out


def reference_arm(args, w):
    """--impl reference: the oracle on the host cores, each step a bounded sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from io_aware_attention_flashattention_b200.inputs import workload_inputs

    inputs = workload_inputs(w)
    budget = args.reference_seconds / max(1, args.steps + args.warmup)
    for i in range(args.warmup):
        oracle_sample(w, budget, rng_seed=i, inputs=inputs)
    flops = secs = 0.0
    rows = threads = 0
    for i in range(args.steps):
        f, t, R, threads = oracle_sample(w, budget, rng_seed=1000 + i, inputs=inputs)
        flops += f
        secs += t
        rows += R
    value = flops / secs / 1e12
    sample = (f"{rows // max(1, args.steps)} random (head, query row) pairs per step of "
              f"{w.name}, all visible keys: oracle forward rows + dQ rows, fp64")
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "impl": "reference",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, int(os.environ.get("WORLD_SIZE", "1"))),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out))
    return 0


# ---------------------------------------------------------------- secondary configurations

# (label, workload, field overrides, window, block-mask density, dropout p). Masked and
# dropout cases use the long workload's shape; a block mask keeps each 128 x 128 block
# with the given probability (numpy seed 77) and always keeps the diagonal blocks.
SECONDARY = [
    ("gpt2_causal_b8h12_n1024_d64", "gpt2_causal_b8h12_n1024_d64", {}, None, None, None),
    ("mid_b1h8_n4096_d128", "mid_b1h8_n4096_d128", {}, None, None, None),
    ("mid_b1h8_n4096_d128_f16", "mid_b1h8_n4096_d128", {"dtype": "f16"}, None, None, None),
    ("stress_causal_b2h16_n8192_d128_qk8", "stress_causal_b2h16_n8192_d128_qk8", {}, None, None,
     None),
    ("long_b1h8_n16384_d128", "long_b1h8_n16384_d128", {}, None, None, None),
    ("long_b1h8_n16384_d128_causal", "long_b1h8_n16384_d128", {"causal": True}, None, None, None),
    ("long_causal_window512", "long_b1h8_n16384_d128", {"causal": True}, (512, 512), None, None),
    ("long_causal_blocks25", "long_b1h8_n16384_d128", {"causal": True}, None, 0.25, None),
    ("long_dropout0.1", "long_b1h8_n16384_d128", {}, None, None, 0.1),
]


def secondary_configs(dev, peak: float, steps: int = 10, warmup: int = 3):
    """Forward and backward TFLOP/s of every SECONDARY case, timed like the main line:
    CUDA events on the launching stream around the forward and around the three
    backward kernels, L2 flushed and the launches queued ahead before each, median of
    ``steps`` steps. FLOPs
    count only the (query, key) pairs the masks keep; the backward is 2.5x the
    forward. Inputs are seeded draws on the device (timing only; the parity tests use
    the host generator)."""
    import dataclasses
    import statistics

    import numpy as np
    import torch

    from io_aware_attention_flashattention_b200 import api
    from io_aware_attention_flashattention_b200.inputs import WORKLOADS, make_inputs_device

    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    out = {}
    for label, wname, over, window, density, p_drop in SECONDARY:
        over = dict(over)
        if over.get("dtype") == "f16":
            over["dtype"] = torch.float16
        w = dataclasses.replace(WORKLOADS[wname], **over)
        q, k, v, do = make_inputs_device(w.B, w.H, w.N, w.d, w.dtype, w.seed, device=dev)
        if w.qk_gain != 1.0:
            q.mul_(w.qk_gain)
            k.mul_(w.qk_gain)
        blocks = None
        if density is not None:
            T = (w.N + 127) // 128
            m = (np.random.default_rng(77).random((T, T)) < density).astype(np.uint8)
            np.fill_diagonal(m, 1)
            blocks = m
        bm = torch.from_numpy(blocks).to(dev) if blocks is not None else None
        drop = (p_drop, 1234, 0) if p_drop is not None else None
        pairs = visible_pairs(w.N, w.causal, window, blocks)
        fwd_f = 4.0 * w.B * w.H * w.d * pairs
        bwd_f = 2.5 * fwd_f
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = api.workspace_for(q)

        def fwd():
            if drop is not None:
                api.fa_forward_dropout(q, k, v, o, lse, w.scale, w.causal, drop, window, bm)
            elif window is not None or bm is not None:
                api.fa_forward_masked(q, k, v, o, lse, w.scale, w.causal, window, bm)
            elif w.dtype == torch.float16:
                api.fa_forward_f16(q, k, v, o, lse, w.scale, w.causal)
            else:
                api.fa_forward(q, k, v, o, lse, w.scale, w.causal)

        def bwd():
            if drop is not None:
                api.fa_backward_dropout(q, k, v, o, do, lse, dq, dk, dv, w.scale, w.causal, ws,
                                        drop, window, bm)
            elif window is not None or bm is not None:
                api.fa_backward_masked(q, k, v, o, do, lse, dq, dk, dv, w.scale, w.causal, ws,
                                       window, bm)
            elif w.dtype == torch.float16:
                api.fa_backward_f16(q, k, v, o, do, lse, dq, dk, dv, w.scale, w.causal, ws)
            else:
                api.fa_backward(q, k, v, o, do, lse, dq, dk, dv, w.scale, w.causal, ws)

        tf, tb = [], []
        for it in range(warmup + steps):
            flush.zero_()
            torch.cuda._sleep(QUEUE_AHEAD_CYCLES)
            e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            e[0].record(stream)
            fwd()
            e[1].record(stream)
            if w.backward:
                flush.zero_()  # the backward starts from a cold L2 too (outside its events)
                torch.cuda._sleep(QUEUE_AHEAD_CYCLES)
                e[2].record(stream)
                bwd()
                e[3].record(stream)
            torch.cuda.synchronize()
            if it >= warmup:
                tf.append(e[0].elapsed_time(e[1]))
                if w.backward:
                    tb.append(e[2].elapsed_time(e[3]))
        if api.fa_get_status() != 0:
            raise SystemExit(f"kernel watchdog fired in {label}")
        ent = {"B": w.B, "H": w.H, "N": w.N, "d": w.d, "dtype": str(w.dtype).split(".")[-1],
               "causal": w.causal, "window": list(window) if window else None,
               "block_density": density, "dropout": p_drop,
               "visible_pairs_per_head": pairs}
        fm = statistics.median(tf)
        ent["fwd_ms"] = fm
        ent["fwd_tflops"] = fwd_f / (fm * 1e-3) / 1e12
        ent["fwd_frac"] = ent["fwd_tflops"] / peak
        if w.backward:
            bm_ms = statistics.median(tb)
            ent["bwd_ms"] = bm_ms
            ent["bwd_tflops"] = bwd_f / (bm_ms * 1e-3) / 1e12
            ent["bwd_frac"] = ent["bwd_tflops"] / peak
        out[label] = ent
        del q, k, v, do, o, lse, dq, dk, dv, ws, bm
    del flush
    return out


# ---------------------------------------------------------------- our arm


def main():
    args = parse()
    from io_aware_attention_flashattention_b200.inputs import WORKLOADS

    w = WORKLOADS[args.workload]
    if args.seq_len is not None and args.seq_len != w.N:
        import dataclasses

        w = dataclasses.replace(w, N=int(args.seq_len),
                                name=f"{w.name.rsplit('_n', 1)[0]}_n{args.seq_len}_d{w.d}")
    if args.impl == "reference":
        return reference_arm(args, w)

    import torch
    import torch.distributed as dist

    from io_aware_attention_flashattention_b200 import api
    from io_aware_attention_flashattention_b200.inputs import make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    # inputs: this rank's replica of the workload (seed offset by rank)
    q, k, v, do = make_inputs(w.B, w.H, w.N, w.d, w.dtype, replica_seed(w, rank), w.qk_gain)
    Q, K, V, dO = (t.to(dev) for t in (q, k, v, do))
    O = torch.empty_like(Q)
    LSE = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    dQ, dK, dV = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V)
    ws = api.workspace_for(Q)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    bf16 = w.dtype == torch.bfloat16
    if not bf16:
        raise SystemExit("the benchmark times the bf16 tensor-core path")

    # the kernels this shape runs (one CTA per item or tile, or their persistent forms)
    plan = api.fa_launch_plan(w.B, w.H, w.N, w.d, w.causal)
    fwd_name = "fa_fwd_persistent_kernel" if plan["fwd_persistent"] else "fa_fwd_kernel"
    bwd_name = "fa_bwd_persistent_kernel" if plan["bwd_persistent"] else "fa_bwd_kernel"
    names = [fwd_name, "fa_bwd_pre_kernel", bwd_name, "fa_bwd_dq_kernel"]
    nev = len(names) + 1

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        api.fa_forward(Q, K, V, O, LSE, w.scale, w.causal)
        if ev is not None:
            ev[1].record(stream)
        api.fa_backward_preprocess(O, dO, LSE, w.scale, w.causal, ws)
        if ev is not None:
            ev[2].record(stream)
        api.fa_backward_main(Q, K, V, dO, dK, dV, w.scale, w.causal, ws)
        if ev is not None:
            ev[3].record(stream)
        api.fa_backward_dq_convert(dQ, w.scale, ws)
        if ev is not None:
            ev[4].record(stream)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if api.fa_get_status() != 0:
        raise SystemExit("kernel watchdog fired during warm-up")

    def timed_region():
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)]
               for _ in range(args.steps)]
        sampler = ClockSampler(torch.cuda.current_device())
        barrier()
        torch.cuda.synchronize()
        sampler.start()
        time.sleep(0.2)  # let the sampler start before the timed region
        t0 = time.perf_counter()
        for s in range(args.steps):
            flush.zero_()
            torch.cuda._sleep(QUEUE_AHEAD_CYCLES)
            step(evs[s])
        torch.cuda.synchronize()
        t1 = time.perf_counter() - t0
        barrier()
        return evs, sampler.stop(), t1

    events, clocks, wall = timed_region()
    # a number taken under a hardware or thermal slowdown, or under a clock lock, is
    # taken again once; every rank takes the same decision (max of the flags)
    rejected = clock_verdict(clocks)
    if max_over_ranks(1.0 if rejected else 0.0, world, dev) > 0:
        first = dict(clocks, rejected=rejected or "another rank's clocks")
        events, clocks, wall = timed_region()
        clocks = dict(clocks, remeasured=True, first_run=first)
    clocks["verdict"] = clock_verdict(clocks) or "ok"
    status = api.fa_get_status()
    per_kernel = [[events[s][i].elapsed_time(events[s][i + 1]) for s in range(args.steps)]
                  for i in range(len(names))]
    step_ms = [events[s][0].elapsed_time(events[s][-1]) for s in range(args.steps)]
    total_ms = max_over_ranks(sum(step_ms), world, dev)

    fwd_f, bwd_f = w.fwd_flops(), w.bwd_flops()
    flops_step = fwd_f + bwd_f
    value = job_throughput(flops_step, world, args.steps, total_ms)

    # per-kernel figures and the dominant kernel's roofline
    BH, N, d = w.B * w.H, w.N, w.d
    npad = (N + 127) // 128 * 128
    kern = {
        fwd_name: {"flops": fwd_f, "bytes": 4 * BH * N * d * 2 + 4 * BH * N},
        "fa_bwd_pre_kernel": {"bytes": 2 * BH * N * d * 2 + 4 * BH * N + 8 * BH * npad
                              + 4 * BH * N * d},
        # reads Q, K, V, dO and L2/D; writes dK, dV; read-modify-write of the fp32 dQ accumulator
        bwd_name: {"flops": bwd_f, "bytes": 6 * BH * N * d * 2 + 8 * BH * npad
                   + 2 * 4 * BH * N * d},
        "fa_bwd_dq_kernel": {"bytes": 4 * BH * N * d + 2 * BH * N * d},
    }
    kernels = {}
    for name, times in zip(names, per_kernel):
        avg = sum(times) / len(times)
        ent = {"avg_ms": avg, "share": sum(times) / total_ms if world == 1 else None}
        if "flops" in kern[name]:
            ent["tflops"] = kern[name]["flops"] / (avg * 1e-3) / 1e12
        ent["gbs"] = kern[name]["bytes"] / (avg * 1e-3) / 1e9
        kernels[name] = ent
    peaks, peak_src = load_peaks()
    dom = max(names, key=lambda n: kernels[n]["avg_ms"])
    if "flops" in kern[dom]:
        achieved = kernels[dom]["tflops"]
        peak = float(peaks["bf16_tflops"])
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak}
    else:
        achieved = kernels[dom]["gbs"]
        peak = float(peaks["hbm_gbs"])
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak}
    roof.update({"traffic": profiled_traffic(dom, w.name), "kernel": dom,
                 "peak_source": f"{peak_src} (burst bf16 GEMM)" if roof["bound"] == "tensor"
                 else f"{peak_src} (copy)"})

    # end to end through the public C-ABI calls with host buffers: every step copies its
    # inputs host -> device and all its results device -> host inside the timed region.
    # Double-buffered on three streams, as a data pipeline would run it: the copy-in of
    # step s+1 and the copy-out of step s-1 overlap the kernels of step s.
    e2e = None
    if not args.no_e2e:
        hq, hk, hv, hdo = (t.pin_memory() for t in (q, k, v, do))
        hO = torch.empty(q.shape, dtype=q.dtype).pin_memory()
        hL = torch.empty((w.B, w.H, w.N), dtype=torch.float32).pin_memory()
        hdQ, hdK, hdV = (torch.empty(q.shape, dtype=q.dtype).pin_memory() for _ in range(3))
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdo))
        d2h = sum(t.numel() * t.element_size() for t in (hO, hL, hdQ, hdK, hdV))
        sets = [dict(Q=Q, K=K, V=V, dO=dO, O=O, LSE=LSE, dQ=dQ, dK=dK, dV=dV, ws=ws)]
        sets.append({name: torch.empty_like(t) for name, t in sets[0].items()})
        s_in, s_run, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))

        def e2e_run(n_steps, start_event):
            in_done, run_done, out_done = [], [], []
            for st in (s_in, s_run, s_out):
                st.wait_event(start_event)
            for i in range(n_steps):
                b = sets[i % 2]
                ev_in, ev_run, ev_out = (torch.cuda.Event() for _ in range(3))
                with torch.cuda.stream(s_in):
                    if i >= 2:  # step i-2's kernels have finished reading this set's inputs
                        s_in.wait_event(run_done[i - 2])
                    for dst, src in ((b["Q"], hq), (b["K"], hk), (b["V"], hv), (b["dO"], hdo)):
                        dst.copy_(src, non_blocking=True)
                    ev_in.record(s_in)
                s_run.wait_event(ev_in)
                if i >= 2:  # step i-2's results have been copied out of this set
                    s_run.wait_event(out_done[i - 2])
                api.fa_forward(b["Q"], b["K"], b["V"], b["O"], b["LSE"], w.scale, w.causal,
                               stream=s_run)
                api.fa_backward(b["Q"], b["K"], b["V"], b["O"], b["dO"], b["LSE"], b["dQ"],
                                b["dK"], b["dV"], w.scale, w.causal, b["ws"], stream=s_run)
                ev_run.record(s_run)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_run)
                    for dst, src in ((hO, b["O"]), (hL, b["LSE"]), (hdQ, b["dQ"]),
                                     (hdK, b["dK"]), (hdV, b["dV"])):
                        dst.copy_(src, non_blocking=True)
                    ev_out.record(s_out)
                in_done.append(ev_in)
                run_done.append(ev_run)
                out_done.append(ev_out)
            for ev in (in_done[-1], run_done[-1], out_done[-1]):
                stream.wait_event(ev)

        warm = torch.cuda.Event()
        warm.record(stream)
        e2e_run(3, warm)
        n_e2e = max(3, min(args.steps, 20))
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_run(n_e2e, e0)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        e2e = {"value": job_throughput(flops_step, world, n_e2e, e_ms), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
               "ms_per_step": e_ms / n_e2e,
               "mode": "two buffer sets, copy-in / kernels / copy-out on three streams"}

    per_config = None
    if world == 1 and not args.no_per_config:
        peaks, _ = load_peaks()
        per_config = secondary_configs(dev, float(peaks["bf16_tflops"]))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f, t, R, threads = oracle_sample(w, args.cpu_seconds)
        cpu = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{R} random (head, query row) pairs of {w.name}, all visible keys: "
                         f"oracle forward rows + dQ rows, fp64, {t:.1f} s",
               "one_thread": oracle_one_thread()}

    if world > 1:
        barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w, world),
        "fwd_tflops": fwd_f / (kernels[names[0]]["avg_ms"] * 1e-3) / 1e12,
        "bwd_tflops": bwd_f / (sum(kernels[n]["avg_ms"] for n in names[1:]) * 1e-3) / 1e12,
        "frac_of_peak": {"fwd": None, "bwd": None, "peak_tflops": float(peaks["bf16_tflops"])},
        "roofline": roof,
        "kernels": kernels,
        "gpu_launches": len(names) * args.steps,
        "clocks": clocks,
        "e2e": e2e,
        "per_config": per_config,
        "cpu_baseline": cpu,
        "watchdog_status": status,
        "wall_s_timed_region": wall,
    }
    pk = float(peaks["bf16_tflops"])
    out["frac_of_peak"]["fwd"] = out["fwd_tflops"] / pk
    out["frac_of_peak"]["bwd"] = out["bwd_tflops"] / pk
    print(json.dumps(out))
    return 0


if __name__ == "__main__":
    sys.exit(main())
