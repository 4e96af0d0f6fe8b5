#!/usr/bin/env python3
"""Benchmark of the int8-LoRA Dense hot path on B200.

One step = forward and backward (dX, dA, dB, dbias of every layer) through
the MNIST MLP stack of int8-LoRA Dense layers: 784 -> 1024, 31 x 1024 ->
1024, 1024 -> 10, ReLU between layers (run in the GEMM epilogues), batch
1024 per GPU, bf16 activations, rank 8, alpha 8 (seeded synthetic data and
weights).  With N
GPUs (torchrun, one process per GPU) every rank runs its own batch and the
LoRA gradients are summed with one NCCL all-reduce per step (weak scaling).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle on
a bounded row sample of the same workload, on the host cores.
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

METRIC = "int8-LoRA Dense fwd+bwd TFLOP/s per step; % of B200 i8/bf16 TC and HBM roofline"
UNIT = "TFLOP/s"
WORKLOAD = "mnist_mlp_stack_33x_int8_lora_dense_bf16_b1024_r8"
L2_FLUSH_BYTES = 384 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def config_dict(n_gpus, batch):
    return {"workload": WORKLOAD, "layers": 33, "dims": "784-1024x32-10", "batch_per_gpu": batch,
            "global_batch": batch * n_gpus, "rank": 8, "alpha": 8.0, "act": "bf16",
            "forward_gemm": "int8 tcgen05", "dx_gemm": "bf16 tcgen05 (int8 dequant in smem)",
            "l2": "flushed between timed steps (384 MiB write)",
            "parallelism": "dp%d" % n_gpus}


# --------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# --------------------------------------------------------------------------
def oracle_stack_sample(rows, specs, data):
    """Runs the oracle's stack on the first `rows` rows; returns seconds."""
    import numpy as np
    import oracle
    layers = []
    for s, L in zip(specs, data["layers"]):
        Wq, sw = oracle.quantize_weight(L["W"])
        layers.append({"Wq": Wq, "sw": sw, "bias": L["bias"], "A": L["A"], "B": L["B"],
                       "alpha": s.alpha})
    X = data["X"][:rows]
    dY = data["dY"][:rows]
    t0 = time.perf_counter()
    oracle.mlp_stack(X, layers, dY, "bf16")
    return time.perf_counter() - t0


def stack_flops(specs, rows):
    tot = 0.0
    for s in specs:
        tot += 4.0 * rows * s.N * s.K
        tot += 2.0 * rows * s.r * (2 * s.K + 2 * s.N) + 2.0 * rows * s.r * (s.K + s.N)
    return tot


def calibrate_rows(specs, data, target_s):
    t = oracle_stack_sample(16, specs, data)
    rows = int(16 * target_s / max(t, 1e-3))
    rows = max(16, min(1024, (rows // 16) * 16))
    return rows


def cpu_baseline(specs, data, target_s=12.0):
    import oracle
    oracle.set_threads(os.cpu_count() or 1)
    rows = calibrate_rows(specs, data, target_s)
    t = oracle_stack_sample(rows, specs, data)
    return {"value": stack_flops(specs, rows) / t / 1e12, "unit": UNIT,
            "cores": oracle.get_threads(), "kind": "oracle",
            "sample": "oracle MLP stack fwd+bwd on the first %d of 1024 rows (all 33 layers), "
                      "%.1f s" % (rows, t)}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    import oracle
    from lora_fine_tuning_qlora_b200 import inputs
    oracle.set_threads(os.cpu_count() or 1)
    specs = inputs.mlp_stack()
    data = inputs.mlp_stack_inputs(specs)
    per_step = max(0.5, min(6.0, 150.0 / max(1, args.steps + args.warmup)))
    rows = calibrate_rows(specs, data, per_step)
    for _ in range(args.warmup):
        oracle_stack_sample(rows, specs, data)
    times = [oracle_stack_sample(rows, specs, data) for _ in range(args.steps)]
    tot = sum(times)
    value = stack_flops(specs, rows) * args.steps / tot / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(world, 1024),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.get_threads(),
                             "kind": "oracle",
                             "sample": "oracle MLP stack fwd+bwd on the first %d of 1024 rows per "
                                       "step (all 33 layers)" % rows},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_id), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100", "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.25)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    p = [x.strip() for x in line.split(",")]
                    if len(p) >= 9:
                        rows.append(p)
            os.unlink(self.path)
        except Exception:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        smax = max((num(r[2]) for r in rows if num(r[2]) is not None), default=None)
        loaded = [v for v in sm if smax and v > 0.5 * smax] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4)
                          if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------
def source_sha(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "lora_fine_tuning_qlora_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_key, src_files):
    """Per-launch DRAM bytes of `kernel_key` from the committed ncu summary,
    if the kernel's source has not changed since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d[kernel_key]
        if e.get("source_sha") == source_sha(*src_files):
            return e["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


def run_ours(args):
    import torch
    from lora_fine_tuning_qlora_b200 import dp, inputs, stack

    rank, local, world = dp.init("nccl")
    if world != args.gpus:
        log("warning: --gpus %d but WORLD_SIZE %d" % (args.gpus, world))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    specs = inputs.mlp_stack()
    data = inputs.mlp_stack_inputs(specs)
    # weak scaling: every rank draws its own batch; the weights are shared
    if world > 1:
        rspecs = [inputs.scaled(s, seed=dp.rank_seed(s.seed, rank)) for s in specs]
        rd = inputs.mlp_stack_inputs(rspecs)
        data = {"layers": data["layers"], "X": rd["X"], "dY": rd["dY"]}
    net = stack.MLPStack.from_inputs(specs, data, device=dev)
    X_dev = torch.from_numpy(data["X"]).to(torch.bfloat16).to(dev)
    dY_dev = torch.from_numpy(data["dY"]).to(torch.bfloat16).to(dev)
    net.X.copy_(X_dev)
    net.dY.copy_(dY_dev)
    # per-kernel events on a few interior 1024x1024 layers only: an event pair
    # serialises the kernel it brackets, so timing every layer slows the step
    mid = [i for i, s in enumerate(specs) if s.K == 1024 and s.N == 1024][3::8]
    events = net.make_events(("gemm_forward", "gemm_dx"), layers=mid)
    net.capture(warmup=1, events=events)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flops = net.flops_per_step()

    def one_step():
        net.replay()
        dp.allreduce_grads(net.grad_flat)

    for _ in range(args.warmup):
        flush.zero_()
        one_step()
    torch.cuda.synchronize()

    # ---------------- timed region (device time, L2 flushed between steps)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    kt = {"gemm_forward": [], "gemm_dx": []}
    gpu_id = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")[local] \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else str(local)
    dp.barrier(dev)
    torch.cuda.synchronize()
    with ClockSampler(gpu_id) as clocks:
        for k in range(args.steps):
            flush.zero_()
            starts[k].record()
            one_step()
            ends[k].record()
            ends[k].synchronize()
            for name in kt:
                kt[name].extend(events[name][i][0].elapsed_time(events[name][i][1]) for i in mid)
        torch.cuda.synchronize()
    dp.barrier(dev)
    total_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    total_ms = dp.max_over_ranks(total_ms, dev)
    value = world * flops * args.steps / (total_ms * 1e-3) / 1e12

    # ---------------- end to end through the public API with host buffers
    Xh = torch.from_numpy(data["X"]).to(torch.bfloat16).pin_memory()
    dYh = torch.from_numpy(data["dY"]).to(torch.bfloat16).pin_memory()
    gh = torch.empty(net.grad_flat.shape, dtype=torch.float32).pin_memory()
    e_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    dp.barrier(dev)
    torch.cuda.synchronize()
    for k in range(args.steps):
        flush.zero_()
        e_s[k].record()
        net.X.copy_(Xh, non_blocking=True)
        net.dY.copy_(dYh, non_blocking=True)
        one_step()
        gh.copy_(net.grad_flat, non_blocking=True)
        e_e[k].record()
    torch.cuda.synchronize()
    dp.barrier(dev)
    e2e_ms = dp.max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(e_s, e_e)), dev)
    e2e_value = world * flops * args.steps / (e2e_ms * 1e-3) / 1e12
    h2d = Xh.numel() * 2 + dYh.numel() * 2
    d2h = gh.numel() * 4

    # ---------------- roofline of the dominant kernel
    peaks, peak_src = load_peaks()
    fwd_ms = statistics.mean(kt["gemm_forward"])
    dx_ms = statistics.mean(kt["gemm_dx"])
    fl_launch = 2.0 * 1024 * 1024 * 1024
    if dx_ms >= fwd_ms:
        dom, ms = "gemm_dx (k3_dx_dequant_kernel, 1024x1024x1024 bf16)", dx_ms
        peak = peaks["bf16_tflops"]
        peak_note = "%s bf16 dense burst" % peak_src
        traffic = profiled_traffic("k3_dx_dequant_kernel", ["k3_dx.cu", "ptx.cuh"])
    else:
        dom, ms = "gemm_forward (k2_gemm_i8_lora_kernel, 1024x1024x1024 int8)", fwd_ms
        peak = 2.0 * peaks["bf16_tflops"]
        peak_note = "%s bf16 dense burst x 2 (nominal int8:bf16 ratio)" % peak_src
        traffic = profiled_traffic("k2_gemm_i8_lora_kernel", ["k2_gemm_i8.cu", "ptx.cuh"])
    achieved = fl_launch / (ms * 1e-3) / 1e12
    roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": traffic, "kernel": dom,
            "peak_source": peak_note, "avg_launch_us": ms * 1e3,
            "launches_timed": len(kt["gemm_dx"]),
            "other": {"gemm_forward_us": fwd_ms * 1e3, "gemm_dx_us": dx_ms * 1e3}}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(specs, data)

    clk = clocks.summary()
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": total_ms / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded; random-init weights of the MNIST MLP shapes)",
                "config": config_dict(world, 1024),
                "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h},
                "gpu_launches": net.launches_per_step() * args.steps,
                "roofline": roof, "cpu_baseline": cpu, "clocks": clk}
        print(json.dumps(line), flush=True)
    net.graph = None
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        log("warmup raised to 3")
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
