#!/usr/bin/env python3
"""Benchmark of the int8-LoRA Dense hot path on B200.

Headline: one step = forward and backward (dX, dA, dB, dbias) of one
int8-LoRA Dense layer with a 4096 x 4096 kernel at M = 16384 tokens, bf16
activations, a rank-4 adapter (alpha 8): the largest single-GPU shape of the
4096-wide layer sweep ("How to fine-tune the 4-bit model?" thread, the
arithmetic-intensity argument for a 4096-wide layer).  With N GPUs (torchrun,
one process per GPU) every rank runs its own 16384 tokens and the LoRA
gradients are summed with one NCCL all-reduce per step (weak scaling).

Beside the headline, the same JSON line carries a ``configs`` list: every
layer of every benchmark workload (the single fp32 layer, the MNIST MLP
stack, the GPT-2 base projections, the Gemma-2B projections at M = 512 and
4096, the 4096-wide layer at M = 16 ... 16384), each with its step time, its
TFLOP/s, the step roofline t_roof / t_measured, and every launch group's
time and fraction of its own roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--no-configs] [--only SUBSTRING]

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle on
a bounded row sample of the headline layer, on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import platform
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "int8-LoRA Dense fwd+bwd TFLOP/s per step; % of B200 i8/bf16 TC and HBM roofline"
UNIT = "TFLOP/s"
HEAD_M = 16384
WORKLOAD = "dense4096_m16384_bf16_r4"
L2_FLUSH_BYTES = 384 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# the kernel each launch group runs at the headline shape (other shapes may
# take the single-CTA GEMMs or the register-resident quantizer)
PART_KERNELS = {
    "quantize_input": ("k1_quantize_rows_kernel", "hbm"),
    "gemm_forward": ("k2_gemm_i8_pair_kernel", "tensor_i8"),
    "lora_grad_dy": ("k4_rank_tc_kernel (dY pass)", "hbm"),
    "gemm_dx": ("k3_dx_pair_kernel", "tensor_bf16"),
    "lora_grad_x": ("k4_rank_tc_kernel (X pass)", "hbm"),
}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"]))}, \
            "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return platform.processor() or "unknown"


def head_config(n_gpus):
    return {"workload": WORKLOAD, "M_per_gpu": HEAD_M, "K": 4096, "N": 4096, "rank": 4,
            "alpha": 8.0, "act": "bf16", "global_batch": HEAD_M * n_gpus, "seq_len": None,
            "forward_gemm": "int8 tcgen05 (K2)", "dx_gemm": "bf16 tcgen05, int8 de-quantized in smem (K3)",
            "l2": "inputs larger than L2, and flushed between timed steps (384 MiB write, then 384 MiB read)",
            "parallelism": "dp%d" % n_gpus}


# --------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# --------------------------------------------------------------------------
def oracle_layer_rows(data, spec, Wq, sw, rows):
    """The oracle's forward + backward of the layer on its first `rows` rows;
    returns seconds."""
    import oracle
    X = data["X"][:rows]
    dY = data["dY"][:rows]
    t0 = time.perf_counter()
    oracle.forward(X, Wq, sw, data["bias"], data["A"], data["B"], spec.alpha)
    oracle.backward(X, dY, Wq, sw, data["A"], data["B"], spec.alpha, want_dx=True, act=spec.act)
    return time.perf_counter() - t0


def layer_flops(M, K, N, r):
    return 4.0 * M * N * K + 2.0 * M * r * (2 * K + 2 * N) + 2.0 * M * r * (K + N)


def oracle_setup(spec, data):
    import oracle
    oracle.set_threads(os.cpu_count() or 1)
    Wq, sw = oracle.quantize_weight(data["W"])
    return Wq, sw


def calibrate_rows(spec, data, Wq, sw, target_s):
    t = oracle_layer_rows(data, spec, Wq, sw, 4)
    rows = int(4 * target_s / max(t, 1e-3))
    return max(4, min(spec.M, rows))


def cpu_baseline(spec, data, target_s=12.0):
    import oracle
    Wq, sw = oracle_setup(spec, data)
    rows = calibrate_rows(spec, data, Wq, sw, target_s)
    t = oracle_layer_rows(data, spec, Wq, sw, rows)
    return {"value": layer_flops(rows, spec.K, spec.N, spec.r) / t / 1e12, "unit": UNIT,
            "cores": oracle.get_threads(), "cpu": cpu_model(), "kind": "oracle",
            "sample": "oracle forward+backward of the %dx%d layer on the first %d of %d rows "
                      "(dA, dB over those rows), %.1f s" % (spec.K, spec.N, rows, spec.M, t)}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    import oracle
    from lora_fine_tuning_qlora_b200 import inputs
    spec = inputs.dense4096(HEAD_M)
    data = inputs.layer_inputs(spec)
    Wq, sw = oracle_setup(spec, data)
    per_step = max(0.5, min(6.0, 150.0 / max(1, args.steps + args.warmup)))
    rows = calibrate_rows(spec, data, Wq, sw, per_step)
    for _ in range(args.warmup):
        oracle_layer_rows(data, spec, Wq, sw, rows)
    times = [oracle_layer_rows(data, spec, Wq, sw, rows) for _ in range(args.steps)]
    tot = sum(times)
    value = layer_flops(rows, spec.K, spec.N, spec.r) * args.steps / tot / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": head_config(world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.get_threads(),
                             "cpu": cpu_model(), "kind": "oracle",
                             "sample": "oracle forward+backward of the 4096x4096 layer on the "
                                       "first %d of %d rows per step" % (rows, HEAD_M)},
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
# roofline arithmetic
# --------------------------------------------------------------------------
def source_sha(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "lora_fine_tuning_qlora_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


TRAFFIC_SOURCES = {
    "k1_quantize_rows_kernel": ["k1_quantize.cu", "ptx.cuh", "tile_epilogue.cuh"],
    "k2_gemm_i8_pair_kernel": ["k2_gemm_i8_pair.cu", "ptx.cuh", "tile_epilogue.cuh"],
    "k3_dx_pair_kernel": ["k3_dx_pair.cu", "dx_common.cuh", "ptx.cuh", "tile_epilogue.cuh"],
    "k4_rank_tc_kernel (dY pass)": ["k4_rank_tc.cu", "ptx.cuh"],
    "k4_rank_tc_kernel (X pass)": ["k4_rank_tc.cu", "ptx.cuh"],
}


def profiled_traffic(kernel, workload):
    """Per-launch DRAM bytes of `kernel` on `workload` from the committed ncu
    summary, if the kernel's sources have not changed since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d[kernel + " @ " + workload]
        if e.get("source_sha") == source_sha(*TRAFFIC_SOURCES[kernel]):
            return e["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


class Roof:
    def __init__(self, peaks):
        self.bw = peaks["hbm_gbs"] * 1e9
        self.bf16 = peaks["bf16_tflops"] * 1e12
        self.i8 = 2.0 * self.bf16  # nominal int8:bf16 dense ratio

    def part(self, name, us, M, K, N, r, e):
        """Achieved rate and fractions of one launch group."""
        from lora_fine_tuning_qlora_b200.step import algorithmic_bytes
        by = algorithmic_bytes(M, K, N, r, e)[name]
        t = us * 1e-6
        kern, bound = PART_KERNELS[name]
        d = {"us": us, "kernel": kern, "bytes": by, "GB/s": by / t / 1e9}
        if bound == "hbm":
            d.update({"bound": "hbm", "frac_hbm": by / t / self.bw})
            d["t_roof_us"] = by / self.bw * 1e6
        else:
            fl = 2.0 * M * N * K
            peak = self.i8 if bound == "tensor_i8" else self.bf16
            d.update({"bound": bound, "T(FL)OP/s": fl / t / 1e12, "frac_tensor": fl / t / peak,
                      "frac_hbm": by / t / self.bw})
            d["t_roof_us"] = max(fl / peak, by / self.bw) * 1e6
        d["frac_roof"] = d["t_roof_us"] / us
        return d

    def step_roof_us(self, M, K, N, r, e):
        """t_roof of one fwd+bwd step: the int8 GEMM and the dX GEMM each at
        the slower of their tensor and byte bounds, plus the byte-bound
        passes (input quantizer, dY pass, X pass) at HBM bandwidth."""
        from lora_fine_tuning_qlora_b200.step import algorithmic_bytes
        b = algorithmic_bytes(M, K, N, r, e)
        fl = 2.0 * M * N * K
        t = max(fl / self.i8, b["gemm_forward"] / self.bw) + max(fl / self.bf16, b["gemm_dx"] / self.bw)
        t += (b["quantize_input"] + b["lora_grad_dy"] + b["lora_grad_x"]) / self.bw
        return t * 1e6


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------
class L2Flush:
    """Between timed steps: writes a 384 MiB buffer (three times L2), then
    reads another one, so that L2 holds only clean lines of data the step does
    not use and the write-back of the written buffer happens before the next
    timed step starts, not inside it."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.max()


def make_step(spec, dev, data=None):
    import torch
    from lora_fine_tuning_qlora_b200 import inputs, qlora, step
    d = data if data is not None else inputs.layer_inputs(spec)
    act = torch.bfloat16 if spec.act == "bf16" else torch.float32
    Wq, sw = qlora.quantize_weight(torch.from_numpy(d["W"]).to(dev))
    bias = torch.from_numpy(d["bias"]).to(dev) if d["bias"] is not None else None
    layer = qlora.Layer(Wq=Wq, sw=sw, bias=bias, A=torch.from_numpy(d["A"]).to(dev),
                        B=torch.from_numpy(d["B"]).to(dev), alpha=spec.alpha, act=act)
    st = step.LayerStep(layer, spec.M, dev)
    st.X.copy_(torch.from_numpy(d["X"]).to(act))
    st.dY.copy_(torch.from_numpy(d["dY"]).to(act))
    return st, d


def time_graph(replay, steps, warmup, flush, between=None):
    """Mean ms of `replay()` over `steps` replays, L2 flushed before each."""
    import torch
    for _ in range(warmup):
        flush()
        replay()
    torch.cuda.synchronize()
    s = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    e = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for k in range(steps):
        flush()
        s[k].record()
        replay()
        e[k].record()
        if between:
            between(k)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in zip(s, e)]


def x_pass_alone(st, steps, flush):
    """Median us of the layer's X pass on its own (one call per replay, L2
    flushed): inside the step it runs beside the dX GEMM, where its events
    span the GEMM too.  G is the step's, left in the workspace."""
    import torch
    from lora_fine_tuning_qlora_b200 import qlora
    L, D, M = st.layer, st.desc, st.M
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    fn = lambda: qlora.qlora_lora_grad_x(D, M, st.X, st.dA, st.ws, s)  # noqa: E731
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fn()
    ms = time_graph(g.replay, steps, 1, flush)
    del g
    return 1e3 * statistics.median(ms)


def overlapped_x(kern, st, steps, flush, M, K, N, r, e, roof):
    """With the X pass beside the dX GEMM, its entry is its time alone, with
    the span of its events inside the step beside it."""
    if st.side is None:
        return kern
    span = kern["lora_grad_x"]["us"]
    kern["lora_grad_x"] = roof.part("lora_grad_x", x_pass_alone(st, steps, flush), M, K, N, r, e)
    kern["lora_grad_x"].update({"beside": "gemm_dx (second stream)", "span_in_step_us": span,
                                "timed": "alone, L2 flushed"})
    return kern


def layer_entry(spec, dev, flush, roof, steps, warmup, data=None):
    """Step time and per-launch-group times of one layer workload."""
    import torch
    from lora_fine_tuning_qlora_b200 import step as step_mod
    st, _ = make_step(spec, dev, data)
    e = 2 if spec.act == "bf16" else 4
    st.capture(warmup=1)
    plain = st.graph
    ms = time_graph(st.replay, steps, warmup, flush)
    ev = st.make_events()
    st.capture(warmup=0, events=ev)
    per = {p: [] for p in step_mod.PARTS}

    def collect(k):
        torch.cuda.synchronize()
        for p in step_mod.PARTS:
            per[p].append(ev[p][0].elapsed_time(ev[p][1]))

    time_graph(st.replay, steps, 1, flush, between=collect)
    step_us = 1e3 * statistics.median(ms)
    M, K, N, r = spec.M, spec.K, spec.N, spec.r
    t_roof = roof.step_roof_us(M, K, N, r, e)
    ent = {"workload": spec.name, "M": M, "K": K, "N": N, "r": r, "act": spec.act,
           "step_us": step_us, "tflops": st.flops() / (step_us * 1e-6) / 1e12,
           "t_roof_us": t_roof, "roof_frac": t_roof / step_us,
           "kernels": overlapped_x({p: roof.part(p, 1e3 * statistics.median(per[p]), M, K, N, r, e)
                                    for p in step_mod.PARTS}, st, steps, flush, M, K, N, r, e, roof)}
    st.graph = None
    del plain
    return ent, st


def mlp_entry(dev, flush, roof, steps, warmup):
    import torch  # noqa: F401
    from lora_fine_tuning_qlora_b200 import inputs, stack
    specs = inputs.mlp_stack()
    data = inputs.mlp_stack_inputs(specs)
    net = stack.MLPStack.from_inputs(specs, data, device=dev)
    import torch as T
    net.X.copy_(T.from_numpy(data["X"]).to(T.bfloat16))
    net.dY.copy_(T.from_numpy(data["dY"]).to(T.bfloat16))
    net.capture(warmup=1)
    ms = time_graph(net.replay, steps, warmup, flush)
    step_us = 1e3 * statistics.median(ms)
    t_roof = sum(roof.step_roof_us(s.M, s.K, s.N, s.r, 2) for s in specs)
    net.graph = None
    return {"workload": "mnist_mlp_stack_33x_b1024_bf16_r8", "layers": len(specs),
            "step_us": step_us, "tflops": net.flops_per_step() / (step_us * 1e-6) / 1e12,
            "t_roof_us": t_roof, "roof_frac": t_roof / step_us,
            "note": "33 layers (784-1024x32-10), ReLU fused in the GEMM epilogues, side-stream "
                    "dB/dA passes, one CUDA graph"}


def merge_entry(st, flush, roof, steps):
    """qlora_merge of a 4096x4096 layer: reads Wq twice, writes Wq' and sw'."""
    import torch
    from lora_fine_tuning_qlora_b200 import qlora
    L = st.layer
    Wq2 = torch.empty_like(L.Wq)
    sw2 = torch.empty_like(L.sw)
    d = L.desc()
    ms = time_graph(lambda: qlora.qlora_merge(d, L.Wq, L.sw, L.A, L.B, Wq2, sw2), steps, 3, flush)
    us = 1e3 * statistics.median(ms)
    by = 2.0 * L.K * L.N + 4.0 * L.N + 4.0 * L.r * (L.K + L.N) + L.K * L.N + 4.0 * L.N
    return {"kernel": "km_merge_kernel", "K": L.K, "N": L.N, "us": us, "bytes": by,
            "GB/s": by / (us * 1e-6) / 1e9, "frac_hbm": by / (us * 1e-6) / roof.bw}


def outlier_entry(spec, dev, flush, roof, steps, warmup):
    """fwd+bwd of the outlier-compensated variant of a layer: the uint8 affine
    kernel rebuilt (with its fp16 outliers) tile by tile in shared memory in
    front of the bf16 tensor cores, in both directions."""
    import torch
    from lora_fine_tuning_qlora_b200 import inputs, qlora
    d = inputs.layer_inputs(spec)
    act = torch.bfloat16
    M, K, N, r = spec.M, spec.K, spec.N, spec.r
    qk = qlora.quantize_outlier(torch.from_numpy(d["W"]).to(dev))
    X = torch.from_numpy(d["X"]).to(act).to(dev)
    dY = torch.from_numpy(d["dY"]).to(act).to(dev)
    A = torch.from_numpy(d["A"]).to(dev)
    B = torch.from_numpy(d["B"]).to(dev)
    bias = torch.from_numpy(d["bias"]).to(dev)
    desc = qlora.desc(K, N, r, spec.alpha, act)
    ws = qlora.workspace(desc, M, dev)
    Y = torch.empty((M, N), dtype=act, device=dev)
    xA = torch.empty((M, r), dtype=torch.float32, device=dev)
    dX = torch.empty((M, K), dtype=act, device=dev)
    dA = torch.empty((K, r), dtype=torch.float32, device=dev)
    dB = torch.empty((r, N), dtype=torch.float32, device=dev)
    db = torch.empty((N,), dtype=torch.float32, device=dev)

    def run():
        qlora.qlora_outlier_forward(desc, M, X, qk, bias, A, B, Y, xA, ws)
        qlora.qlora_outlier_backward(desc, M, X, dY, qk, A, B, xA, dX, dA, dB, db, ws)

    run()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    ms = time_graph(g.replay, steps, warmup, flush)
    step_us = 1e3 * statistics.median(ms)
    e = 2
    fl = 2.0 * M * N * K
    # both GEMMs on bf16 tensor cores; the forward reads X, the uint8 codes and
    # writes Y; the input pass reads X and writes xA
    from lora_fine_tuning_qlora_b200.step import algorithmic_bytes
    b = algorithmic_bytes(M, K, N, r, e)
    fwd_bytes = M * K * e + K * N + M * N * e + 4.0 * (N + M * r + r * N)
    t_roof = (max(fl / roof.bf16, fwd_bytes / roof.bw) + max(fl / roof.bf16, b["gemm_dx"] / roof.bw)
              + (M * K * e + 4.0 * M * r + b["lora_grad_dy"] + b["lora_grad_x"]) / roof.bw) * 1e6
    flops = 4.0 * M * N * K + 2.0 * M * r * (2 * K + 2 * N) + 2.0 * M * r * (K + N)
    del g
    return {"workload": spec.name.replace("gpt2_", "gpt2_outlier_"), "M": M, "K": K, "N": N, "r": r,
            "act": "bf16", "outliers": qk.count, "step_us": step_us,
            "tflops": flops / (step_us * 1e-6) / 1e12, "t_roof_us": t_roof,
            "roof_frac": t_roof / step_us,
            "note": "outlier-compensated uint8 kernel, rebuilt in shared memory before bf16 "
                    "tensor cores in both directions"}


def float8_entry(name, M, K, N, dev, flush, roof, steps, warmup):
    """One training step of a float8 Dense layer ("Introduce float8 training"):
    three delayed-scaling quantizations (E4M3 input and kernel, E5M2 output
    gradient), the forward, dX and dW GEMMs on float8 tensor cores, and the
    bias gradient.  The float8 peak is twice the measured bf16 peak (the
    nominal dense ratio)."""
    import torch
    from lora_fine_tuning_qlora_b200.float8 import Float8Dense
    g = torch.Generator(device="cpu").manual_seed(M + K + N)
    W = (torch.randn(K, N, generator=g) * 0.02).to(dev)
    bias = torch.zeros(N, device=dev)
    X = torch.randn(M, K, generator=g).to(torch.bfloat16).to(dev)
    dY = (torch.randn(M, N, generator=g) * 1e-2).to(torch.bfloat16).to(dev)
    lay = Float8Dense(W, bias, torch.bfloat16, history_len=1024)

    def run():
        _, ctx = lay.forward(X)
        lay.backward(ctx, dY)

    run()
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        run()
    ms = time_graph(gr.replay, steps, warmup, flush)
    step_us = 1e3 * statistics.median(ms)
    fl = 6.0 * M * N * K
    peak8 = 2.0 * roof.bf16
    # bytes: the three tensors read, their codes written twice (row-major and
    # transposed), the GEMMs' outputs
    by = 2.0 * (M * K + M * N) + 4.0 * K * N + 2.0 * (M * K + K * N + M * N) + 2.0 * (M * N + M * K) + 4.0 * K * N
    t_roof = (fl / peak8 + by / roof.bw) * 1e6
    del gr
    return {"workload": name, "M": M, "K": K, "N": N, "act": "bf16", "recipe": "float8 (E4M3 x, W; E5M2 dY)",
            "step_us": step_us, "tflops": fl / (step_us * 1e-6) / 1e12, "t_roof_us": t_roof,
            "roof_frac": t_roof / step_us, "frac_fp8_peak": fl / (step_us * 1e-6) / peak8}


def all_configs(dev, flush, roof, steps, only):
    from lora_fine_tuning_qlora_b200 import inputs
    specs = [inputs.single_fp32()] + inputs.gpt2_base() + inputs.gemma_2b(512) + \
        inputs.gemma_2b(4096) + [inputs.dense4096(m) for m in inputs.DENSE4096_M if m != HEAD_M]
    out = []
    if not only or "mlp" in only:
        out.append(mlp_entry(dev, flush, roof, steps, 3))
    merge = None
    for s in specs:
        if only and only not in s.name:
            continue
        ent, st = layer_entry(s, dev, flush, roof, steps, 3)
        if s.name.startswith("dense4096") and merge is None:
            merge = merge_entry(st, flush, roof, steps)
        out.append(ent)
        del st
    for s in inputs.gpt2_base():
        if only and only not in s.name.replace("gpt2_", "gpt2_outlier_"):
            continue
        out.append(outlier_entry(s, dev, flush, roof, steps, 3))
    for name, M, K, N in (("float8_gpt2_mlp_up_4096x768x3072", 4096, 768, 3072),
                          ("float8_dense4096_16384x4096x4096", 16384, 4096, 4096)):
        if only and only not in name:
            continue
        out.append(float8_entry(name, M, K, N, dev, flush, roof, steps, 3))
    return out, merge


def run_ours(args):
    import torch
    from lora_fine_tuning_qlora_b200 import dp, inputs, step as step_mod

    rank, local, world = dp.init("nccl")
    if world != args.gpus:
        log("warning: --gpus %d but WORLD_SIZE %d" % (args.gpus, world))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks, peak_src = load_peaks()
    roof = Roof(peaks)

    # weak scaling: every rank draws its own tokens; the weights are shared
    spec = inputs.dense4096(HEAD_M)
    data = inputs.layer_inputs(spec)
    if world > 1:
        rd = inputs.layer_inputs(inputs.scaled(spec, seed=dp.rank_seed(spec.seed, rank)))
        data = dict(data, X=rd["X"], dY=rd["dY"])
    st, _ = make_step(spec, dev, data)
    flops = st.flops()
    flush = L2Flush(dev)
    # the timed graph brackets every launch group with events on the launching
    # stream; the kernels are long enough (tens to hundreds of us) that the
    # event pairs cost them little
    ev = st.make_events()
    st.capture(warmup=1, events=ev)

    def one_step():
        st.replay()
        dp.allreduce_grads(st.grad_flat)

    for _ in range(args.warmup):
        flush()
        one_step()
    torch.cuda.synchronize()

    # ---------------- timed region (device time, L2 flushed between steps)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    per = {p: [] for p in step_mod.PARTS}
    gpu_id = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")[local] \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else str(local)
    dp.barrier(dev)
    torch.cuda.synchronize()
    with ClockSampler(gpu_id) as clocks:
        for k in range(args.steps):
            flush()
            starts[k].record()
            one_step()
            ends[k].record()
            # the graph's events hold the latest replay: read them before the next
            ends[k].synchronize()
            for p in step_mod.PARTS:
                per[p].append(ev[p][0].elapsed_time(ev[p][1]))
        torch.cuda.synchronize()
    dp.barrier(dev)
    total_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    total_ms = dp.max_over_ranks(total_ms, dev)
    value = world * flops * args.steps / (total_ms * 1e-3) / 1e12

    # ---------------- end to end through the public API with host buffers
    # Every step copies its inputs from pinned host memory and reads its
    # gradients back, as a training loop with a prefetching loader would: two
    # sets of device buffers (two captured steps of the same layer) take
    # turns, and the copies of step k + 1 run on a copy stream while step k
    # computes.  The timed region runs from the first copy to the last read;
    # the inputs (256 MiB a step) are larger than L2, so no flush is added.
    Xh = torch.from_numpy(data["X"]).to(torch.bfloat16).pin_memory()
    dYh = torch.from_numpy(data["dY"]).to(torch.bfloat16).pin_memory()
    gh = [torch.empty(st.grad_flat.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    st.graph = None
    st.capture(warmup=1)
    st2 = step_mod.LayerStep(st.layer, spec.M, dev)
    st2.capture(warmup=1)
    sts = (st, st2)
    main, cs = torch.cuda.current_stream(), torch.cuda.Stream()
    copied = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    e_s = [torch.cuda.Event(enable_timing=True)]
    e_e = [torch.cuda.Event(enable_timing=True)]
    dp.barrier(dev)
    torch.cuda.synchronize()
    e_s[0].record(main)
    cs.wait_stream(main)
    for k in range(args.steps):
        b = k % 2
        sk = sts[b]
        with torch.cuda.stream(cs):
            if k >= 2:
                cs.wait_event(done[b])  # step k - 2 is done with these buffers
            sk.X.copy_(Xh, non_blocking=True)
            sk.dY.copy_(dYh, non_blocking=True)
            copied[b].record(cs)
        main.wait_event(copied[b])
        sk.replay()
        dp.allreduce_grads(sk.grad_flat)
        gh[b].copy_(sk.grad_flat, non_blocking=True)
        done[b].record(main)
    e_e[0].record(main)
    torch.cuda.synchronize()
    dp.barrier(dev)
    st2.graph = None
    e2e_ms = dp.max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(e_s, e_e)), dev)
    e2e_value = world * flops * args.steps / (e2e_ms * 1e-3) / 1e12
    h2d = Xh.numel() * 2 + dYh.numel() * 2
    d2h = gh[0].numel() * 4

    # ---------------- roofline of the dominant kernel and of the step
    M, K, N, r = spec.M, spec.K, spec.N, spec.r
    kern = {p: roof.part(p, 1e3 * statistics.mean(per[p]), M, K, N, r, 2) for p in step_mod.PARTS}
    kern = overlapped_x(kern, st, args.steps, flush, M, K, N, r, 2, roof)
    # the dominant launch group by its own time (the X pass's events, beside
    # the dX GEMM, are not its duration)
    dom = max((p for p in kern if "span_in_step_us" not in kern[p]), key=lambda p: kern[p]["us"])
    kd = kern[dom]
    name, bound = PART_KERNELS[dom]
    if bound == "hbm":
        roofline = {"bound": "hbm", "achieved": kd["GB/s"], "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": kd["frac_hbm"]}
    else:
        peak = peaks["bf16_tflops"] * (2.0 if bound == "tensor_i8" else 1.0)
        roofline = {"bound": "tensor", "achieved": kd["T(FL)OP/s"], "peak": peak,
                    "unit": "TFLOP/s", "frac": kd["frac_tensor"]}
    roofline.update({
        "traffic": profiled_traffic(name, WORKLOAD), "kernel": "%s (%s, %dx%dx%d bf16)" % (name, dom, M, K, N),
        "peak_source": "%s %s" % (peak_src, "HBM copy" if bound == "hbm" else
                                  "bf16 dense burst" + (" x 2 (nominal int8:bf16 ratio)"
                                                        if bound == "tensor_i8" else "")),
        "avg_launch_us": kd["us"], "algorithmic_per_launch": kd["bytes"] if bound == "hbm"
        else 2.0 * M * N * K, "launches_timed": len(per[dom])})
    t_roof = roof.step_roof_us(M, K, N, r, 2)
    ms_step = total_ms / args.steps
    step_roof = {"t_roof_us": t_roof, "t_measured_us": 1e3 * ms_step,
                 "frac": t_roof / (1e3 * ms_step),
                 "rule": "max(2MNK/P_i8, bytes_fwd/BW) + max(2MNK/P_bf16, bytes_dx/BW) + "
                         "(bytes_quantize + bytes_dY_pass + bytes_X_pass)/BW"}

    configs, merge = None, None
    if rank == 0 and world == 1 and not args.no_configs:
        st.graph = None
        configs, merge = all_configs(dev, flush, roof, args.config_steps, args.only)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(spec, data)

    clk = clocks.summary()
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms_step, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded; random-init weights of the 4096x4096 layer)",
                "config": head_config(world),
                "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h},
                "gpu_launches": st.launches_per_step() * args.steps,
                "roofline": roofline, "step_roofline": step_roof, "kernels": kern,
                "cpu_baseline": cpu, "clocks": clk,
                "peaks": dict(peaks, source=peak_src),
                "merge": merge, "configs": configs}
        print(json.dumps(line), flush=True)
    st.graph = None
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
    ap.add_argument("--no-configs", action="store_true", help="headline only")
    ap.add_argument("--config-steps", type=int, default=10, help="timed steps per config layer")
    ap.add_argument("--only", default="", help="time only the config layers whose name contains this")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        log("warmup raised to 3")
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
