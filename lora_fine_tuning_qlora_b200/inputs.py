"""Seeded synthetic inputs for the int8-LoRA Dense layer workloads.

This module only draws random numbers and shapes them; it holds none of the
layer's arithmetic (no quantization, no matmul).  Both the CUDA path (through
``bench.py`` and the GPU tests) and the CPU oracle (through the tests) take
their inputs from here, so the two sides see the same values.

Every tensor is drawn in fp32 with ``numpy.random.Generator(PCG64(seed))`` in
a fixed order.  For bf16 workloads the activations (X, dY) are then rounded to
bf16 once (``torch`` RNE conversion); the fp32 widening of those bf16 values is
what the oracle receives, and the bf16 tensor is what the GPU receives.  The
kernel W, bias and the LoRA factors A and B stay fp32 (LoRA weights are kept
in fp32, keras-llm-light README, "Weights quantization").

Workload shapes follow the pages:
  * single fp32 layer 64x784 -> 128 (MNIST MLP width, "Introduce QLoRA-like
    technique", benchmark.py);
  * the MNIST MLP stack at batch 1024 (same page, benchmark.py and Results);
  * GPT-2 base projections at 32 x 128 tokens ("Parameter-efficient
    fine-tuning of GPT-2 with LoRA"; Keras PR 19356 GPT-2 table);
  * Gemma-2B projections (keras-llm-light README, block memory table);
  * a 4096 x 4096 layer with a rank-4 adapter ("How to fine-tune the 4-bit
    model?" thread).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Dict, List, Optional

import numpy as np


@dataclass(frozen=True)
class LayerSpec:
    """Shape and value recipe of one int8-LoRA Dense layer.

    M tokens, K in_features, N out_features, rank r, LoRA alpha.  ``act`` is
    the activation dtype ("f32" or "bf16").  The ``*_dist`` strings name the
    distributions drawn by :func:`layer_inputs`.
    """

    name: str
    M: int
    K: int
    N: int
    r: int
    alpha: float
    act: str = "bf16"
    x_dist: str = "normal"          # normal | uniform01
    w_dist: str = "glorot"          # glorot | normal002 | normal002_outliers | student_t3
    a_dist: str = "he_uniform"      # he_uniform | uniform_inv_sqrt_k | uniform_1_64
    b_std: float = 0.01
    bias_dist: str = "normal001"    # normal001 | zeros | none
    dy_std: float = 1.0
    seed: int = 0

    @property
    def c(self) -> float:
        return float(self.alpha) / float(self.r)


# --------------------------------------------------------------------------
# distributions
# --------------------------------------------------------------------------
def _draw_w(rng, spec: LayerSpec) -> np.ndarray:
    K, N = spec.K, spec.N
    if spec.w_dist == "glorot":
        lim = math.sqrt(6.0 / (K + N))
        return rng.uniform(-lim, lim, size=(K, N)).astype(np.float32)
    if spec.w_dist == "normal002":
        return rng.normal(0.0, 0.02, size=(K, N)).astype(np.float32)
    if spec.w_dist == "normal002_outliers":
        w = rng.normal(0.0, 0.02, size=(K, N))
        n_out = max(1, int(round(0.001 * K * N)))
        idx = rng.choice(K * N, size=n_out, replace=False)
        w.reshape(-1)[idx] *= 20.0
        return w.astype(np.float32)
    if spec.w_dist == "student_t3":
        w = rng.standard_t(3.0, size=(K, N)) * 0.02
        return np.clip(w, -1.0, 1.0).astype(np.float32)
    raise ValueError(spec.w_dist)


def _draw_a(rng, spec: LayerSpec) -> np.ndarray:
    K, r = spec.K, spec.r
    if spec.a_dist == "he_uniform":
        # VarianceScaling(scale=sqrt(5), mode="fan_in", distribution="uniform")
        lim = math.sqrt(3.0 * math.sqrt(5.0) / K)
    elif spec.a_dist == "uniform_inv_sqrt_k":
        lim = 1.0 / math.sqrt(K)
    elif spec.a_dist == "uniform_1_64":
        lim = 1.0 / 64.0
    else:
        raise ValueError(spec.a_dist)
    return rng.uniform(-lim, lim, size=(K, r)).astype(np.float32)


def _draw_x(rng, spec: LayerSpec, M: int) -> np.ndarray:
    if spec.x_dist == "normal":
        return rng.standard_normal(size=(M, spec.K), dtype=np.float32)
    if spec.x_dist == "uniform01":
        return rng.random(size=(M, spec.K), dtype=np.float32)
    raise ValueError(spec.x_dist)


def round_to_act(a: np.ndarray, act: str) -> np.ndarray:
    """fp32 array -> fp32 array holding the values the activation dtype stores."""
    if act == "f32":
        return np.ascontiguousarray(a, np.float32)
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)
    return t.to(torch.float32).numpy()


def layer_inputs(spec: LayerSpec, with_x: bool = True, with_dy: bool = True) -> Dict[str, np.ndarray]:
    """Draw W, bias, A, B (always) and X, dY (optional) for one layer.

    Returns fp32 numpy arrays; X and dY already hold activation-dtype values.
    The draw order is fixed: W, bias, A, B, X, dY.
    """
    rng = np.random.Generator(np.random.PCG64(spec.seed))
    W = _draw_w(rng, spec)
    if spec.bias_dist == "normal001":
        bias = rng.normal(0.0, 0.01, size=(spec.N,)).astype(np.float32)
    elif spec.bias_dist == "zeros":
        bias = np.zeros((spec.N,), np.float32)
    else:
        bias = None
    A = _draw_a(rng, spec)
    B = rng.normal(0.0, spec.b_std, size=(spec.r, spec.N)).astype(np.float32) \
        if spec.b_std > 0 else np.zeros((spec.r, spec.N), np.float32)
    out = {"W": W, "bias": bias, "A": A, "B": B}
    if with_x:
        out["X"] = round_to_act(_draw_x(rng, spec, spec.M), spec.act)
    if with_dy:
        dy = rng.standard_normal(size=(spec.M, spec.N), dtype=np.float32) * np.float32(spec.dy_std)
        out["dY"] = round_to_act(dy, spec.act)
    return out


# --------------------------------------------------------------------------
# the workloads
# --------------------------------------------------------------------------
def single_fp32() -> LayerSpec:
    """One fp32 layer, X [64,784], W [784,128], rank 4, alpha 4, seed 0."""
    return LayerSpec("single_fp32_64x784x128", M=64, K=784, N=128, r=4, alpha=4.0,
                     act="f32", x_dist="normal", w_dist="glorot",
                     a_dist="uniform_inv_sqrt_k", b_std=0.01, bias_dist="normal001",
                     dy_std=1.0, seed=0)


def mlp_stack(batch: int = 1024, hidden: int = 1024, depth: int = 31,
              r: int = 8, alpha: float = 8.0, act: str = "bf16") -> List[LayerSpec]:
    """The MNIST MLP: 784 -> hidden, depth x (hidden -> hidden), hidden -> 10."""
    dims = [784] + [hidden] * (depth + 1) + [10]
    specs = []
    for i in range(len(dims) - 1):
        specs.append(LayerSpec("mlp%d_%dx%d" % (i, dims[i], dims[i + 1]),
                               M=batch, K=dims[i], N=dims[i + 1], r=r, alpha=alpha,
                               act=act, x_dist="uniform01", w_dist="glorot",
                               a_dist="uniform_inv_sqrt_k", b_std=0.01,
                               bias_dist="zeros", dy_std=1.0, seed=100 + i))
    return specs


def mlp_stack_inputs(specs: List[LayerSpec]) -> Dict[str, object]:
    """Per-layer W/bias/A/B plus the stack input X and the top gradient dY."""
    layers = [layer_inputs(s, with_x=False, with_dy=False) for s in specs]
    first = layer_inputs(specs[0], with_x=True, with_dy=False)
    last = layer_inputs(specs[-1], with_x=False, with_dy=True)
    return {"layers": layers, "X": first["X"], "dY": last["dY"]}


def gpt2_base(M: int = 4096) -> List[LayerSpec]:
    shapes = [("qkv", 768, 2304), ("attn_out", 768, 768), ("mlp_up", 768, 3072),
              ("mlp_down", 3072, 768)]
    return [LayerSpec("gpt2_%s_%dx%dx%d" % (n, M, K, N), M=M, K=K, N=N, r=4, alpha=32.0,
                      act="bf16", x_dist="normal", w_dist="normal002_outliers",
                      a_dist="he_uniform", b_std=0.01, bias_dist="normal001",
                      dy_std=1e-2, seed=200 + i)
            for i, (n, K, N) in enumerate(shapes)]


def gemma_2b(M: int = 512) -> List[LayerSpec]:
    shapes = [("q", 2048, 2048), ("k", 2048, 256), ("v", 2048, 256), ("o", 2048, 2048),
              ("gate", 2048, 16384), ("up", 2048, 16384), ("down", 16384, 2048)]
    return [LayerSpec("gemma_%s_%dx%dx%d" % (n, M, K, N), M=M, K=K, N=N, r=4, alpha=32.0,
                      act="bf16", x_dist="normal", w_dist="normal002",
                      a_dist="he_uniform", b_std=0.01, bias_dist="normal001",
                      dy_std=1.0, seed=300 + i)
            for i, (n, K, N) in enumerate(shapes)]


def dense4096(M: int) -> LayerSpec:
    return LayerSpec("dense4096_%dx4096x4096" % M, M=M, K=4096, N=4096, r=4, alpha=8.0,
                     act="bf16", x_dist="normal", w_dist="student_t3",
                     a_dist="uniform_1_64", b_std=0.01, bias_dist="normal001",
                     dy_std=1.0, seed=400 + M)


DENSE4096_M = (16, 64, 256, 1024, 4096, 16384)


def scaled(spec: LayerSpec, **kw) -> LayerSpec:
    """A copy of ``spec`` with some fields replaced (e.g. a smaller M)."""
    return replace(spec, **kw)
