#!/usr/bin/env python
"""Benchmark of the SVDQuant W4A4 + rank-32 linear (NVFP4) on the FLUX fused-QKV layer
(M = 4608 tokens, K = 3072, N = 9216, rank 32) on B200.

One step = one pass of the hot path on one batch: kernel 1 (smoothing + 4-bit quantization +
bf16 down projection) and kernel 2 (block-scaled 4-bit GEMM + up projection + bias).  Three
independent copies of the layer (inputs, outputs, workspace and prepared weights; ~400 MB, over
3x the 126 MB L2) are used in rotation, so no step finds its operands in L2.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle instead.
Multi-GPU (torchrun): every rank runs its own replica of the layer (weak scaling, no
data-path collective); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A4+rank-32 linear TFLOP/s & % FP4 peak; low-rank overhead % on one B200"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = "flux_qkv_4608x3072x9216_r32"
FP4_PER_BF16 = 4.0  # nominal dense ratio: 9 PFLOP/s fp4 / 2.25 PFLOP/s bf16
INT8_PER_BF16 = 2.0  # nominal dense ratio: 4.5 POP/s int8 / 2.25 PFLOP/s bf16 (INT4 runs on kind::i8)
KERNEL_LAUNCHES = 240  # per-kernel timing loop (and each variant of the overhead legs)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = [os.path.join(ROOT, "w4a4_rank_corrected_smooth_b200", "csrc", f)
                  for f in ("kernels.cu", "ptx.cuh", "layout.h")]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=30)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--precision", default="nvfp4")
    ap.add_argument("--sets", type=int, default=3, help="rotating copies of the layer")
    ap.add_argument("--no-extras", action="store_true", help="skip overhead, e2e and CPU-baseline legs")
    ap.add_argument("--no-clocks", action="store_true", help="do not sample nvidia-smi (profiling runs)")
    ap.add_argument("--sweep", action="store_true",
                    help="one JSON line per FLUX-shaped layer and per point of the M x rank sweep (not the driver's line)")
    ap.add_argument("--sweep-filter", default=None,
                    help="with --sweep: only the workloads whose name matches this regular expression, no legs")
    ap.add_argument("--leg", choices=["w4a16", "mlp_pair", "qkv_norm_rope"], default=None,
                    help="run one auxiliary leg alone and print its JSON line (not the driver's line; profiling)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    """sha256 of the kernel sources' code (kernels.cu and the headers it compiles with): comments,
    trailing blanks and blank lines removed, so a comment edit does not orphan the ncu counters
    while any change to the code does."""
    import re

    text = ""
    for path in KERNEL_SOURCES:
        with open(path, encoding="utf-8") as f:
            text += f.read() + "\n"
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = []
    for line in text.splitlines():
        code = re.sub(r"//.*$", "", line) if '"' not in line else line  # keep lines with strings intact
        code = code.rstrip()
        if code:
            lines.append(code)
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()


def stored_traffic(kernel: str, workload: str):
    """dram bytes per launch from a committed ncu summary, if taken on the current kernel source."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
        e = d[kernel][workload]
        if e.get("source_sha256") == kernel_source_hash():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ---------------------------------------------------------------- clocks


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.tmp = tempfile.NamedTemporaryFile(prefix="svdq_clk_", suffix=".csv", delete=False)
        self.proc = None
        self.device_index = device_index
        self.t_start = self.t_stop = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", str(self.device_index)], stdout=self.tmp, stderr=subprocess.DEVNULL)
            time.sleep(1.0)
        except Exception:
            self.proc = None

    def mark(self, start: bool):
        if start:
            self.t_start = time.time()
        else:
            self.t_stop = time.time()

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        self.tmp.close()
        rows = []
        try:
            with open(self.tmp.name) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
        finally:
            os.unlink(self.tmp.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        # nvidia-smi rows carry no timestamps here: keep the loaded ones (power above idle).
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        pw = [num(r[3]) for r in rows]
        pmax = max([p for p in pw if p is not None] or [0.0])
        loaded = [r for r, p in zip(rows, pw) if p is not None and p >= 0.5 * pmax] or rows
        sm = [num(r[1]) for r in loaded if num(r[1]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in loaded:
            for name, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": num(loaded[0][2]),
                "reasons": sorted(reasons), "samples": len(loaded), "power_w_max": pmax}


# ---------------------------------------------------------------- helpers


def hold_gpu(stream, us: float):
    """Keeps the GPU busy for about ``us`` microseconds (a spin kernel on ``stream``), so that the
    host can queue the launches of a timed region before the region starts: the timed region then
    measures the GPU, not the host's launch latency."""
    import torch

    with torch.cuda.stream(stream):
        torch.cuda._sleep(int(min(max(us, 20.0), 50000.0) * 2000))  # ~2 GHz SM clock


def bf16_device(x_bits, device):
    import numpy as np
    import torch

    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).view(torch.bfloat16).to(device)


def dist_info():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, world: int) -> float:
    """Max of a per-rank float over all ranks (identity at world size 1)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(flops_per_step: float, steps: int, local_ms: float, world: int):
    """Whole-job throughput (TFLOP/s) of `world` replicas that each ran `steps` steps: the work of
    all ranks over the slowest rank's time.  Returns (value, slowest_ms)."""
    slowest = max_over_ranks(local_ms, world)
    return world * flops_per_step * steps / (slowest / 1e3) / 1e12, slowest


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def workload_config(spec, precision: str, world: int, sets: int) -> dict:
    """The ``config`` object of the JSON line; both arms print the same one for one workload."""
    return {"workload": spec.name, "M": spec.M, "K": spec.K, "N": spec.N, "rank": spec.rank,
            "precision": precision, "parallelism": f"replicas x{world}",
            "l2": f"{sets} rotating copies of X/Y/workspace/weights (> 3x L2), no flush"}


def oracle_cpu_baseline(X, ops, precision, spec, budget_s: float = 10.0):
    """Times the oracle's forward on a row sample of the workload (all N, all K)."""
    import numpy as np
    from oracle import svdq_oracle as O

    try:
        from threadpoolctl import threadpool_info

        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count()])
    except Exception:
        cores = os.cpu_count()
    def timed(rows):
        t0 = time.perf_counter()
        O.linear(X[:rows], ops, precision)
        return time.perf_counter() - t0

    # t(rows) ~ a + b * rows (a: per-call dequantization of W); size the sample for the budget.
    t_small, t_big = timed(64), timed(512)
    slope = max((t_big - t_small) / 448.0, 1e-9)
    fixed = max(t_small - 64 * slope, 0.0)
    rows = int((budget_s - fixed) / slope)
    rows = max(64, min(spec.M, rows // 64 * 64))
    dt = timed(rows)
    flops = 2 * rows * spec.N * spec.K + 2 * rows * spec.rank * (spec.K + spec.N)
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": int(cores), "kind": "oracle",
            "sample": f"oracle.linear (fp64) on rows 0..{rows - 1} of {spec.M} (all {spec.N} outputs, K={spec.K}), "
                      f"one call, {dt:.2f} s wall"}


# ---------------------------------------------------------------- reference arm


def run_reference(args):
    """The CPU oracle, as it stands, on the same workload/metric: each step is oracle.linear on a
    block of output rows x columns sized so that warm-up + steps end within a few minutes."""
    import numpy as np

    import synth
    from oracle import svdq_oracle as O

    world, rank, _ = dist_info()
    if rank != 0:
        return
    spec = synth.get(args.workload)
    X = synth.activations_bf16(spec)
    W = synth.weight_bf16(spec)
    b = synth.bias_bf16(spec)
    a = synth.act_absmax(X)
    ops = O.prepare(W, b, a, args.precision, spec.rank)
    try:
        from threadpoolctl import threadpool_info

        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count()])
    except Exception:
        cores = os.cpu_count()
    budget = 150.0 / max(1, args.steps + args.warmup)
    rows, cols = 16, 64

    def sliced(c0, cols):
        d = dict(ops)
        d["codes_w"] = ops["codes_w"][c0:c0 + cols]
        d["scales_w"] = ops["scales_w"][c0:c0 + cols]
        d["L2"] = ops["L2"][:, c0:c0 + cols]
        d["bias"] = ops["bias"][c0:c0 + cols]
        return d

    t0 = time.perf_counter()
    O.linear(X[:rows], sliced(0, cols), args.precision)
    dt = time.perf_counter() - t0
    while dt * 4 < budget and (rows < spec.M or cols < spec.N):
        if cols < spec.N:
            cols = min(spec.N, cols * 2)
        else:
            rows = min(spec.M, rows * 2)
        t0 = time.perf_counter()
        O.linear(X[:rows], sliced(0, cols), args.precision)
        dt = time.perf_counter() - t0
    flops = 2 * rows * cols * spec.K + 2 * rows * spec.rank * (spec.K + cols)
    rng = np.random.default_rng(0)
    for i in range(args.warmup):
        r0 = int(rng.integers(0, spec.M - rows + 1))
        c0 = int(rng.integers(0, (spec.N - cols) // 8 + 1)) * 8
        O.linear(X[r0:r0 + rows], sliced(c0, cols), args.precision)
    t0 = time.perf_counter()
    for i in range(args.steps):
        r0 = int(rng.integers(0, spec.M - rows + 1))
        c0 = int(rng.integers(0, (spec.N - cols) // 8 + 1)) * 8
        O.linear(X[r0:r0 + rows], sliced(c0, cols), args.precision)
    total = time.perf_counter() - t0
    value = flops * args.steps / total / 1e12
    sample = f"per step: oracle.linear on a {rows} x {cols} block of Y (K={spec.K}) of {spec.M} x {spec.N}"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(spec, args.precision, world, args.sets),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": int(cores), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- our arm


def time_loop(layers, sets, steps, stream, sample_every: int = 8):
    """Runs `steps` steps rotating over `sets`; returns (total_ms, mean k1 ms, mean k2 ms).

    The total comes from events before the first and after the last step.  The per-kernel
    durations come from events around the two kernels of every `sample_every`-th step only: an
    event between the kernels would keep kernel 2's prologue from overlapping kernel 1's tail
    (programmatic dependent launch), so most steps run without one."""
    import torch

    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    samples = []
    hold_gpu(stream, 40.0 * steps)
    start.record(stream)
    for i in range(steps):
        lin = layers[i % len(layers)]
        X, Y, ws = sets[i % len(sets)]
        M = X.shape[0]
        sampled = i % sample_every == sample_every // 2 or steps < sample_every
        if sampled:
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            ev[0].record(stream)
        lin.svdq_quant_down(X, M, X.stride(0), ws, ws.numel(), stream)
        if sampled:
            ev[1].record(stream)
        lin.svdq_gemm_up(M, Y, Y.stride(0), ws, ws.numel(), stream)
        if sampled:
            ev[2].record(stream)
            samples.append(ev)
    end.record(stream)
    torch.cuda.synchronize()
    total = start.elapsed_time(end)
    k1 = sum(e[0].elapsed_time(e[1]) for e in samples) / len(samples)
    k2 = sum(e[1].elapsed_time(e[2]) for e in samples) / len(samples)
    return total, k1, k2


def kernel_times(layers, sets, stream, launches: int = 200):
    """Per-kernel durations from their own loop of ``launches`` steps over the rotating sets, with
    events around each kernel of every step (the event between the kernels keeps kernel 2 from
    overlapping kernel 1's tail, so each duration is the kernel's own).  Returns a dict with the
    mean and median of each kernel in ms and the number of launches each."""
    import statistics as st

    import torch

    time_loop(layers, sets, 3, stream, sample_every=1)
    k1s, k2s = [], []
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    evs = []
    hold_gpu(stream, 100.0 * launches)
    start.record(stream)
    for i in range(launches):
        lin = layers[i % len(layers)]
        X, Y, ws = sets[i % len(sets)]
        M = X.shape[0]
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record(stream)
        lin.svdq_quant_down(X, M, X.stride(0), ws, ws.numel(), stream)
        ev[1].record(stream)
        lin.svdq_gemm_up(M, Y, Y.stride(0), ws, ws.numel(), stream)
        ev[2].record(stream)
        evs.append(ev)
    end.record(stream)
    torch.cuda.synchronize()
    for ev in evs:
        k1s.append(ev[0].elapsed_time(ev[1]))
        k2s.append(ev[1].elapsed_time(ev[2]))
    return {"quant_down": sum(k1s) / len(k1s), "gemm": sum(k2s) / len(k2s),
            "quant_down_median": st.median(k1s), "gemm_median": st.median(k2s), "launches": launches}


def qkv_norm_rope_leg(layers, sets, spec, stream, steps):
    """The grouped QKV operator with RMS normalization of Q and K and the rotary embedding fused
    into kernel 2's epilogue, against the plain forward on the same layer copies and buffers:
    whole steps (both kernels), ``steps`` each, events before the first and after the last."""
    import numpy as np
    import torch

    import synth
    import w4a4_rank_corrected_smooth_b200 as S

    D = 128
    dev = sets[0][0].device
    cos, sin = synth.rope_tables(spec.M, D)
    rope_rows = torch.from_numpy(np.stack([cos, sin], axis=-1).reshape(spec.M, D).astype(np.float32)).to(dev)
    # packed once (a model computes its rotary table once per resolution and reuses it in every layer)
    rope = torch.empty(S.svdq_rope_packed_size(spec.M, D) // 4, dtype=torch.float32, device=dev)
    S.svdq_pack_rope(rope_rows, spec.M, D, rope, rope.numel() * 4, stream)
    gq = torch.from_numpy(synth.rms_norm_weight(D, 1)).to(dev)
    gk = torch.from_numpy(synth.rms_norm_weight(D, 2)).to(dev)

    def run(fused):
        for i in range(steps):
            lin = layers[i % len(layers)]
            X, Y, ws = sets[i % len(sets)]
            if fused:
                lin.svdq_linear_forward_qkv_norm_rope(X, spec.M, X.stride(0), Y, Y.stride(0), gq, gk, 1e-6, rope, D,
                                                      ws, ws.numel(), stream)
            else:
                lin.svdq_linear_forward(X, spec.M, X.stride(0), Y, Y.stride(0), ws, ws.numel(), stream)

    out = {}
    for fused in (False, True, False, True):
        run(fused)  # warm-up of this variant
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        hold_gpu(stream, 40.0 * steps)
        a.record(stream)
        run(fused)
        b.record(stream)
        b.synchronize()
        key = "ms_per_step_fused" if fused else "ms_per_step_plain"
        out[key] = min(out.get(key, float("inf")), a.elapsed_time(b) / steps)
    out["overhead_pct"] = 100.0 * (out["ms_per_step_fused"] / out["ms_per_step_plain"] - 1.0)
    out.update({"heads": spec.N // (3 * D), "head_dim": D, "eps": 1e-6, "steps": steps,
                "what": "QKV layer + RMS norm of Q and K + rotary turn of channel pairs, in kernel 2's epilogue"})
    return out


def e2e_pipelined(lin, X, spec, sets, stream, steps: int = 30):
    """Per-step time of host X -> forward -> host Y through svdq_linear_forward, pipelined over a
    copy-in stream, the compute stream and a copy-out stream with two device buffer sets (events
    order the reuse of each buffer).  Returns (ms per step, steps, H2D bytes, D2H bytes)."""
    import numpy as np
    import torch

    Xh = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16).pin_memory()
    Yh = [torch.empty((spec.M, spec.N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    bufs = [sets[0]]
    if len(sets) > 1:
        bufs.append(sets[1])
    else:
        X0, Y0, w0 = sets[0]
        bufs.append((torch.empty_like(X0), torch.empty_like(Y0), torch.empty_like(w0)))
    s_in = torch.cuda.Stream(device=stream.device)
    s_out = torch.cuda.Stream(device=stream.device)

    def run(n):
        ev_in = [None] * n
        ev_fw = [None] * n
        ev_out = [None] * n
        for i in range(n):
            Xd, Yd, ws = bufs[i % 2]
            if i >= 2:
                s_in.wait_event(ev_fw[i - 2])  # Xd of step i-2 has been consumed
            with torch.cuda.stream(s_in):
                Xd.copy_(Xh, non_blocking=True)
            ev_in[i] = torch.cuda.Event()
            ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            if i >= 2:
                stream.wait_event(ev_out[i - 2])  # Yd of step i-2 has been copied out
            lin.svdq_linear_forward(Xd, spec.M, spec.K, Yd, spec.N, ws, ws.numel(), stream)
            ev_fw[i] = torch.cuda.Event()
            ev_fw[i].record(stream)
            s_out.wait_event(ev_fw[i])
            with torch.cuda.stream(s_out):
                Yh[i % 2].copy_(Yd, non_blocking=True)
            ev_out[i] = torch.cuda.Event()
            ev_out[i].record(s_out)
        return ev_out[n - 1]

    run(3)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    last = run(steps)
    s_out.wait_event(last)
    e1.record(s_out)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps, steps, int(Xh.numel() * 2), int(Yh[0].numel() * 2)


def unfused_comparator(lin, layers, sets, layers0, sets0, steps, stream, k2_bare_ms):
    """The same layer with the low-rank branch unfused (the pages' naive version, for context):
    kernel 1 and kernel 2 of the rank-0 layer, plus a separate down projection that reads X again
    (one cuBLAS GEMM with the smoothing folded into L1: X (diag(1/lambda) L1)) and a separate up
    projection that reads and rewrites Y (Y += T L2, one cuBLAS GEMM with beta = 1).  Not the
    product: a timing comparator only.  All three variants are timed as whole steps."""
    import numpy as np
    import torch

    dev = sets[0][0].device
    ops = lin.export_weights()
    il = torch.from_numpy(ops["inv_lambda"].astype(np.float32)).to(dev)
    L1 = bf16_device(ops["L1"], dev).float()
    L1s = (il[:, None] * L1).to(torch.bfloat16).contiguous()
    L2 = bf16_device(ops["L2"], dev).contiguous()
    Ts = [torch.empty((x.shape[0], L1s.shape[1]), dtype=torch.bfloat16, device=dev) for (x, _, _) in sets]

    def unfused_steps(n):
        for i in range(n):
            l0 = layers0[i % len(layers0)]
            X, Y, ws = sets0[i % len(sets0)]
            T = Ts[i % len(Ts)]
            M = X.shape[0]
            l0.svdq_quant_down(X, M, X.stride(0), ws, ws.numel(), stream)
            torch.mm(X, L1s, out=T)
            l0.svdq_gemm_up(M, Y, Y.stride(0), ws, ws.numel(), stream)
            Y.addmm_(T, L2)

    def fused_steps(lays, sts, n):
        for i in range(n):
            l = lays[i % len(lays)]
            X, Y, ws = sts[i % len(sts)]
            M = X.shape[0]
            l.svdq_quant_down(X, M, X.stride(0), ws, ws.numel(), stream)
            l.svdq_gemm_up(M, Y, Y.stride(0), ws, ws.numel(), stream)

    def timed(fn):
        fn(3)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        hold_gpu(stream, 60.0 * steps)
        e0.record(stream)
        fn(steps)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    t_unfused = timed(unfused_steps)
    t_fused = timed(lambda n: fused_steps(layers, sets, n))
    t_bare = timed(lambda n: fused_steps(layers0, sets0, n))
    return {"ms_step": {"fused_rank": t_fused, "unfused_rank": t_unfused, "rank0": t_bare},
            "fused_pct_of_bare_gemm": 100.0 * (t_fused - t_bare) / k2_bare_ms,
            "unfused_pct_of_bare_gemm": 100.0 * (t_unfused - t_bare) / k2_bare_ms,
            "fused_pct_of_bare_layer": 100.0 * (t_fused - t_bare) / t_bare,
            "unfused_pct_of_bare_layer": 100.0 * (t_unfused - t_bare) / t_bare,
            "comparator": "down projection X (diag(1/lambda) L1) and up projection Y += T L2 as separate cuBLAS GEMMs"}


W4A16_SHAPES = [(1, 3072, 18432), (2, 3072, 18432), (4, 3072, 18432), (1, 3072, 9216)]


def w4a16_leg(dev, stream, peaks, peak_src, launches: int = 200):
    """The W4A16 layer on FLUX's modulation projections (one token per image: M rows of K = 3072
    into N = 6*3072 or 3*3072).  ``launches`` launches back to back on one stream, rotating over
    enough copies of the layer's weights that their total exceeds twice the L2 cache (so every
    launch streams its weights from HBM, with no flush kernel in between), CUDA events around the
    whole run; the time per launch includes the gap between consecutive launches.  Weight-only
    4-bit layers of this size are bound by HBM, so the roofline is the measured copy bandwidth."""
    import numpy as np
    import torch

    import synth
    import w4a4_rank_corrected_smooth_b200 as S

    out = {}
    prepared = {}
    l2_bytes = 126 << 20
    for (M, K, N) in W4A16_SHAPES:
        if (K, N) not in prepared:
            for lins_, _ in prepared.values():
                for l_ in lins_:
                    l_.close()
            prepared.clear()
            spec = synth.custom(f"flux_modulation_{K}x{N}", M=8, K=K, N=N, rank=0, seed=N)
            X8 = synth.activations_bf16(spec)
            lin = S.SVDQLinear(synth.weight_bf16(spec), synth.bias_bf16(spec), synth.act_absmax(X8), "w4a16", 0,
                               device=dev.index)
            wbytes = N * K // 2 + 4 * N * (K // 64)
            ncopies = max(2, -(-2 * l2_bytes // wbytes))
            prepared[(K, N)] = ([lin] + [lin.clone() for _ in range(ncopies - 1)], X8)
        lins, X8 = prepared[(K, N)]
        Xd = bf16_device(np.ascontiguousarray(X8[:M]), dev)
        Ys = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(2)]
        for i in range(2 * len(lins)):
            lins[i % len(lins)].svdq_linear_forward(Xd, M, K, Ys[i % 2], N, None, 0, stream)
        hold_gpu(stream, 30.0 * launches)  # the launches are queued before the timed region starts
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(launches):
            lins[i % len(lins)].svdq_linear_forward(Xd, M, K, Ys[i % 2], N, None, 0, stream)
        e1.record(stream)
        e1.synchronize()
        S.svdq_get_device_error(stream)
        ms = e0.elapsed_time(e1) / launches
        nbytes = N * K // 2 + 4 * N * (K // 64) + 2 * M * K + 2 * M * N + 4 * K + 4 * N
        gbs = nbytes / (ms / 1e3) / 1e9
        out[f"{M}x{K}x{N}"] = {"us": ms * 1e3, "algorithmic_bytes_per_launch": nbytes, "achieved_gbs": gbs,
                               "frac": gbs / peaks["hbm_gbs"], "weight_copies": len(lins)}
    for lins_, _ in prepared.values():
        for l_ in lins_:
            l_.close()
    timing = f"{launches} launches back to back over rotating weight copies (> 2x L2), events around the run"
    return {"kernel": "w4a16_kernel", "bound": "hbm", "peak_gbs": peaks["hbm_gbs"], "peak_source": peak_src,
            "timing": timing, "shapes": out}


def run_ours(args):
    import numpy as np
    import torch

    import synth
    import w4a4_rank_corrected_smooth_b200 as S

    world, rank, local = dist_info()
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    S.svdq_check_device(local)
    stream = torch.cuda.current_stream(dev)
    spec = synth.get(args.workload)
    X = synth.activations_bf16(spec)
    W = synth.weight_bf16(spec)
    b = synth.bias_bf16(spec)
    a = synth.act_absmax(X)
    lin = S.SVDQLinear(W, b, a, args.precision, spec.rank, device=local)
    layers = [lin] + [lin.clone() for _ in range(args.sets - 1)]
    Xd = bf16_device(X, dev)
    sets = []
    for s in range(args.sets):
        perm = torch.randperm(spec.M, generator=torch.Generator().manual_seed(s)).to(dev)
        Xs = Xd if s == 0 else Xd[perm].contiguous()
        Ys = torch.empty((spec.M, spec.N), dtype=torch.bfloat16, device=dev)
        ws = lin.new_workspace(spec.M)
        sets.append((Xs, Ys, ws))
    peaks, peak_src = load_peaks()

    sampler = ClockSampler(int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local])
                           if os.environ.get("CUDA_VISIBLE_DEVICES") else local)
    if not args.no_clocks:
        sampler.start()
    time_loop(layers, sets, max(3, args.warmup), stream)
    S.svdq_get_device_error(stream)
    barrier(world)
    torch.cuda.synchronize()
    sampler.mark(True)
    total_ms, _, _ = time_loop(layers, sets, args.steps, stream)
    torch.cuda.synchronize()
    sampler.mark(False)
    barrier(world)
    # Per-kernel durations (roofline of each kernel): their own loop of KERNEL_LAUNCHES steps,
    # whatever --steps is, with clocks still sampled.
    kt = kernel_times(layers, sets, stream, KERNEL_LAUNCHES)
    k1_ms, k2_ms = kt["quant_down"], kt["gemm"]
    clocks = sampler.stop() if not args.no_clocks else None
    S.svdq_get_device_error(stream)
    flops = spec.flops
    value, total_ms = weak_scaling_value(flops, args.steps, total_ms, world)
    k2_flops = spec.flops_4bit + 2 * spec.M * spec.rank * spec.N
    k2_tflops = k2_flops / (k2_ms / 1e3) / 1e12
    nvfp4 = args.precision == "nvfp4"
    ratio = FP4_PER_BF16 if nvfp4 else INT8_PER_BF16
    tensor_kind = "fp4" if nvfp4 else "int8"
    # The GEMM's own tensor dtype.  Each kernel is timed alone for tens of microseconds at the
    # maximum clock, so the burst figure is its peak; the sustained one (seconds-long loops under
    # the power cap, at a lower clock) is reported beside it.
    fp4_peak_sustained = peaks["bf16_tflops_sustained"] * ratio
    fp4_peak_burst = peaks["bf16_tflops"] * ratio
    sfx = "" if nvfp4 else "_int4"
    k1_bytes = (2 * spec.M * spec.K + spec.M * spec.K // 2 + spec.M * spec.K // 16 + 2 * spec.K * spec.rank
                + 2 * spec.M * spec.rank)
    k2_bytes = (spec.M * spec.K // 2 + spec.M * spec.K // 16 + spec.N * spec.K // 2 + spec.N * spec.K // 16
                + 2 * spec.M * spec.rank + 2 * spec.N * spec.rank + 4 * spec.N + 2 * spec.M * spec.N)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4" if args.precision == "nvfp4" else "int4",
        "data": "synthetic (seeded FLUX-shaped activations with 0.5% x30 outlier channels, W ~ N(0, 0.02))",
        "config": workload_config(spec, args.precision, world, args.sets),
        "tensor_peak_frac": value / world / fp4_peak_burst,
        "kernel_ms": kt,
        "roofline": {"bound": "tensor", "achieved": k2_tflops, "peak": fp4_peak_burst, "unit": "TFLOP/s",
                     "frac": k2_tflops / fp4_peak_burst, "traffic": stored_traffic("gemm" + sfx, spec.name),
                     "kernel": "gemm_nvfp4_kernel" if nvfp4 else "gemm_int4_kernel",
                     "peak_source": f"{peak_src} bf16 burst x {ratio:g} (nominal {tensor_kind}/bf16)",
                     "frac_of_sustained_peak": k2_tflops / fp4_peak_sustained,
                     "sustained_peak": fp4_peak_sustained,
                     "timing": f"mean of {kt['launches']} launches, events around each kernel",
                     "algorithmic_flops_per_launch": k2_flops},
        "quant_down_roofline": {"bound": "hbm", "achieved": k1_bytes / (k1_ms / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                                "unit": "GB/s", "frac": k1_bytes / (k1_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                                "traffic": stored_traffic("quant_down" + sfx, spec.name),
                                "algorithmic_bytes_per_launch": k1_bytes},
        "gemm_algorithmic_bytes_per_launch": k2_bytes,
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
    }

    if not args.no_extras:
        # Low-rank overhead: the same layer prepared with rank 0, timed the same way.
        lin0 = S.SVDQLinear(W, b, a, args.precision, 0, device=local)
        layers0 = [lin0] + [lin0.clone() for _ in range(args.sets - 1)]
        sets0 = [(x, y, lin0.new_workspace(spec.M)) for (x, y, _) in sets]
        n_over = KERNEL_LAUNCHES
        kt0 = kernel_times(layers0, sets0, stream, n_over)
        ktr = kernel_times(layers, sets, stream, n_over)
        k1_0, k2_0, k1_r, k2_r = kt0["quant_down"], kt0["gemm"], ktr["quant_down"], ktr["gemm"]
        S.svdq_get_device_error(stream)
        over = (k1_r + k2_r - k1_0 - k2_0)
        line["lowrank_overhead_pct"] = 100.0 * over / k2_0
        line["lowrank_overhead_detail"] = {
            "rank": spec.rank, "ms_rank": {"quant_down": k1_r, "gemm": k2_r},
            "ms_rank0": {"quant_down": k1_0, "gemm": k2_0},
            "pct_of_bare_gemm": 100.0 * over / k2_0, "pct_of_bare_layer": 100.0 * over / (k1_0 + k2_0),
            "timing": f"means of {n_over} launches of each kernel per variant, events around each kernel"}
        line["lowrank_overhead_unfused"] = unfused_comparator(lin, layers, sets, layers0, sets0, n_over, stream, k2_0)
        if nvfp4 and spec.N % (3 * 128) == 0:
            line["qkv_norm_rope"] = qkv_norm_rope_leg(layers, sets, spec, stream, n_over)
        for l0 in layers0:
            l0.close()
        # End to end through the public API: every step copies X from pinned host memory to the
        # device, runs the forward and copies Y back to pinned host memory.  Steps are pipelined
        # over three streams and two device buffer sets (the copy in of step i+1 and the copy out
        # of step i-1 overlap the forward of step i), as a serving loop would run them.
        e2e_ms, n_e2e, h2d, d2h = e2e_pipelined(lin, X, spec, sets, stream)
        e2e_ms = max_over_ranks(e2e_ms, world)
        line["e2e"] = {"value": world * flops / (e2e_ms / 1e3) / 1e12, "unit": UNIT,
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "ms_per_step": e2e_ms, "steps": n_e2e,
                       "pipeline": "3 streams (copy in, forward, copy out), 2 device buffer sets"}
        if world == 1:
            line["cpu_baseline"] = oracle_cpu_baseline(X, lin.export_weights(), args.precision, spec)
            try:  # an auxiliary leg: its failure is reported in the line, not fatal to it
                line["w4a16_modulation"] = w4a16_leg(dev, stream, peaks, peak_src)
            except Exception as exc:  # noqa: BLE001
                line["w4a16_modulation"] = {"error": f"{type(exc).__name__}: {exc}"}
    for l in layers:
        l.close()
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_sweep(args):
    """Times every FLUX-shaped layer (QKV, MLP pair, DiT block) and the M x rank sweep at K = N =
    3072 on one GPU: one JSON line each, with the step time (both kernels, whole steps), the
    per-kernel times, TFLOP/s over the algorithmic flops, and the low-rank overhead against the
    same layer prepared with rank 0.  Two rotating copies of X/Y/workspace per point."""
    import numpy as np
    import torch

    import synth
    import w4a4_rank_corrected_smooth_b200 as S

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    S.svdq_check_device(0)
    stream = torch.cuda.current_stream(dev)
    peaks, peak_src = load_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16  # kernels timed alone: the burst figure
    names = ["flux_qkv_4608x3072x9216_r32", "flux_mlp_up_4608x3072x12288_r32", "flux_mlp_down_4608x12288x3072_r32",
             "dit_qkv_mlp_in_16896x3072x21504_r32", "dit_out_16896x15360x3072_r32"]
    names += [f"sweep_{M}x3072x3072_r{r}" for r in (0, 16, 32, 64, 128) for M in (256, 1024, 4096, 16384)]
    if args.sweep_filter:
        import re
        names = [n for n in names if re.search(args.sweep_filter, n)]
    prepared = {}
    xcache = {}
    for name in names:
        if not name.startswith("sweep"):
            xcache.clear()
        spec = synth.get(name)
        key = (spec.K, spec.N, spec.rank, name.split("_")[0] if name.startswith("sweep") else name)
        if key not in prepared:
            calib = synth.activations_bf16(spec.with_rows(min(spec.M, 4096)))
            W = synth.weight_bf16(spec)
            b = synth.bias_bf16(spec)
            a = synth.act_absmax(calib)
            for l_, l0_ in prepared.values():
                l_.close()
                l0_.close()
            prepared.clear()
            prepared[key] = (S.SVDQLinear(W, b, a, args.precision, spec.rank, device=0),
                             S.SVDQLinear(W, b, a, args.precision, 0, device=0))
        lin, lin0 = prepared[key]
        xkey = spec.name.rsplit("_r", 1)[0]  # the sweep's points of one M share X
        if xkey not in xcache:
            xcache[xkey] = bf16_device(synth.activations_bf16(spec), dev)
        Xd = xcache[xkey]
        sets = []
        for s_ in range(2):
            Xs = Xd if s_ == 0 else Xd.roll(1, 0).contiguous()
            sets.append((Xs, torch.empty((spec.M, spec.N), dtype=torch.bfloat16, device=dev), lin.new_workspace(spec.M)))
        steps = max(20, min(400, int(2e12 / max(spec.flops, 1))))
        time_loop([lin], sets, 5, stream)
        t, _, _ = time_loop([lin], sets, steps, stream)
        ms = t / steps
        kt = kernel_times([lin], sets, stream, KERNEL_LAUNCHES)
        k1, k2 = kt["quant_down"], kt["gemm"]
        sets0 = [(x, y, lin0.new_workspace(spec.M)) for (x, y, _) in sets]
        time_loop([lin0], sets0, 5, stream)
        t0, _, _ = time_loop([lin0], sets0, steps, stream)
        ms0 = t0 / steps
        kt0 = kernel_times([lin0], sets0, stream, KERNEL_LAUNCHES)
        k10, k20 = kt0["quant_down"], kt0["gemm"]
        unfused = None
        if spec.rank > 0:  # the pages' naive branch (separate down and up projections), same point
            unfused = unfused_comparator(lin, [lin], sets, [lin0], sets0, max(steps, 50), stream, k20)
        S.svdq_get_device_error(stream)
        k2_flops = spec.flops_4bit + 2 * spec.M * spec.rank * spec.N
        out = {"sweep": True, "workload": spec.name, "M": spec.M, "K": spec.K, "N": spec.N, "rank": spec.rank,
               "precision": args.precision, "steps": steps, "ms_per_step": ms,
               "tflops": spec.flops / (ms / 1e3) / 1e12,
               "kernel_ms": {"quant_down": k1, "gemm": k2},
               "gemm_tflops": k2_flops / (k2 / 1e3) / 1e12,
               "gemm_frac_fp4_peak": k2_flops / (k2 / 1e3) / 1e12 / fp4_peak,
               "ms_per_step_rank0": ms0, "kernel_ms_rank0": {"quant_down": k10, "gemm": k20},
               "lowrank_overhead_pct_of_bare_gemm": 100.0 * (k1 + k2 - k10 - k20) / k20,
               "lowrank_overhead_pct_of_bare_gemm_whole_steps": 100.0 * (ms - ms0) / k20,
               "unfused": unfused,
               "kernel_launches_timed": KERNEL_LAUNCHES,
               "peak": {"fp4_tflops": fp4_peak, "source": f"{peak_src} bf16 burst x {FP4_PER_BF16:g}"}}
        print(json.dumps(out), flush=True)
        del sets, sets0
    for l, l0 in prepared.values():
        l.close()
        l0.close()
    if args.sweep_filter:
        return
    print(json.dumps({"sweep": True, "w4a16_modulation": w4a16_leg(dev, stream, peaks, peak_src)}), flush=True)
    print(json.dumps({"sweep": True, "mlp_pair": mlp_pair_leg(dev, stream, peaks)}), flush=True)


def mlp_pair_leg(dev, stream, peaks, steps: int = 200):
    """FLUX's MLP pair (4608 x 3072 -> 12288 -> GELU -> 3072, rank 32, NVFP4) three ways: fused
    (the up layer's epilogue emits the down layer's 4-bit operands; the hidden activation never
    reaches memory), GELU-fused (the up layer's GELU-output forward, then the down layer's
    forward on the hidden activation) and unfused (up forward writing bf16 Y, GELU by torch, down
    forward); whole steps timed with CUDA events, two rotating buffer sets."""
    import torch

    import synth
    import w4a4_rank_corrected_smooth_b200 as S

    up_spec = synth.get("flux_mlp_up_4608x3072x12288_r32")
    down_spec = synth.get("flux_mlp_down_4608x12288x3072_r32")
    X = synth.activations_bf16(up_spec)
    up = S.SVDQLinear(synth.weight_bf16(up_spec), synth.bias_bf16(up_spec), synth.act_absmax(X), "nvfp4", 32,
                      device=dev.index)
    calib = synth.activations_bf16(down_spec.with_rows(4096))
    down = S.SVDQLinear(synth.weight_bf16(down_spec), synth.bias_bf16(down_spec), synth.act_absmax(calib), "nvfp4", 32,
                        device=dev.index)
    M = up_spec.M
    sets = []
    for s_ in range(2):
        Xd = bf16_device(X, dev) if s_ == 0 else bf16_device(X, dev).roll(1, 0).contiguous()
        sets.append({"X": Xd, "Y": torch.empty((M, down.N), dtype=torch.bfloat16, device=dev),
                     "H": torch.empty((M, up.N), dtype=torch.bfloat16, device=dev),
                     "ws_up": up.new_workspace(M), "ws_down": down.new_workspace(M),
                     "mid": torch.empty(S.svdq_mlp_workspace_size(up, down, M), dtype=torch.uint8, device=dev)})

    def fused(b):
        S.svdq_mlp_forward(up, down, b["X"], M, b["X"].stride(0), b["Y"], b["Y"].stride(0), b["ws_up"],
                           b["ws_up"].numel(), b["mid"], b["mid"].numel(), stream)

    def gelu_fused(b):
        up.svdq_linear_forward_gelu(b["X"], M, b["X"].stride(0), b["H"], b["H"].stride(0), b["ws_up"],
                                    b["ws_up"].numel(), stream)
        down.svdq_linear_forward(b["H"], M, b["H"].stride(0), b["Y"], b["Y"].stride(0), b["ws_down"],
                                 b["ws_down"].numel(), stream)

    def unfused(b):
        up.svdq_linear_forward(b["X"], M, b["X"].stride(0), b["H"], b["H"].stride(0), b["ws_up"], b["ws_up"].numel(),
                               stream)
        torch.nn.functional.gelu(b["H"], out=b["H"])
        down.svdq_linear_forward(b["H"], M, b["H"].stride(0), b["Y"], b["Y"].stride(0), b["ws_down"],
                                 b["ws_down"].numel(), stream)

    out = {}
    for name, fn in (("unfused", unfused), ("fused", fused), ("gelu_fused", gelu_fused)) * 2:
        for i in range(10):
            fn(sets[i % 2])
        a = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        hold_gpu(stream, 80.0 * steps)
        a.record(stream)
        for i in range(steps):
            fn(sets[i % 2])
        e.record(stream)
        e.synchronize()
        out[f"ms_{name}"] = min(out.get(f"ms_{name}", float("inf")), a.elapsed_time(e) / steps)
    S.svdq_get_device_error(stream)
    flops = up_spec.flops + down_spec.flops
    out.update({"tflops_fused": flops / (out["ms_fused"] / 1e3) / 1e12,
                "tflops_gelu_fused": flops / (out["ms_gelu_fused"] / 1e3) / 1e12,
                "tflops_unfused": flops / (out["ms_unfused"] / 1e3) / 1e12,
                "speedup": out["ms_unfused"] / out["ms_fused"],
                "speedup_gelu_fused": out["ms_unfused"] / out["ms_gelu_fused"], "steps": steps,
                "unfused_gelu": "torch.nn.functional.gelu on the bf16 hidden tensor (a library kernel)"})
    up.close()
    down.close()
    return out


def run_leg(args):
    """One auxiliary leg on GPU 0, alone (used to profile its kernel): the W4A16 modulation
    projections, FLUX's MLP pair (fused against unfused) or the fused QKV operator."""
    import torch

    import w4a4_rank_corrected_smooth_b200 as S

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    S.svdq_check_device(0)
    stream = torch.cuda.current_stream(dev)
    peaks, peak_src = load_peaks()
    if args.leg == "w4a16":
        out = w4a16_leg(dev, stream, peaks, peak_src, launches=max(3, args.steps))
    elif args.leg == "mlp_pair":
        out = mlp_pair_leg(dev, stream, peaks, steps=max(3, args.steps))
    else:  # the fused QKV operator on the FLUX QKV layer, against the plain forward
        import synth

        spec = synth.get(DEFAULT_WORKLOAD)
        X = synth.activations_bf16(spec)
        lin = S.SVDQLinear(synth.weight_bf16(spec), synth.bias_bf16(spec), synth.act_absmax(X), "nvfp4", spec.rank,
                           device=0)
        Xd = bf16_device(X, dev)
        sets = [(Xd, torch.empty((spec.M, spec.N), dtype=torch.bfloat16, device=dev), lin.new_workspace(spec.M))]
        out = qkv_norm_rope_leg([lin], sets, spec, stream, max(3, args.steps))
        lin.close()
    print(json.dumps({"leg": args.leg, args.leg: out}), flush=True)


def main():
    args = parse_args()
    world, _, _ = dist_info()
    if world != args.gpus and not (world == 1 and args.gpus == 1):
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    elif args.leg:
        run_leg(args)
    elif args.sweep:
        run_sweep(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
