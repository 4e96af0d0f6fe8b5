"""One int8-LoRA Dense layer, forward and backward, as a replayable step.

The layer computes (QLoRA-like PR, "Introduce QLoRA-like technique"; GPT-2
LoRA notebook, "LoRA equation"):

    forward   Xq, sx, xA = quantize(X), X . A            (K1)
              Y = (Xq Wq^T) sx sw + bias + c xA B          (K2)
    backward  G = dY B^T, dB = c xA^T dY, dbias = sum dY   (dY pass)
              dX = dY (Wq sw)^T + c G A^T                  (K3)
              dA = c X^T G                                 (X pass)

``LayerStep`` owns the device buffers of one layer at M tokens and issues the
five launch groups through the step-level C-ABI calls, so a step can be
captured into a CUDA graph and replayed.  Optional CUDA events bracket each
launch group for per-kernel timing.

dX and dA both need only G (and the inputs), so after the dY pass the X pass
runs on a second stream beside the dX GEMM (an event fork and join, which a
CUDA graph captures as two branches): its CTAs take the SMs the GEMM leaves
idle, in the GEMM's last partial wave of tiles or beside a GEMM too small to
fill the GPU.
"""
from __future__ import annotations

from typing import Dict, Optional, Tuple

import torch

from . import qlora

# the launch groups of one step, in issue order
PARTS = ("quantize_input", "gemm_forward", "lora_grad_dy", "gemm_dx", "lora_grad_x")


class LayerStep:
    def __init__(self, layer: qlora.Layer, M: int, device="cuda", overlap_x: Optional[bool] = None):
        dev = torch.device(device)
        self.layer = layer
        self.M = M
        self.desc = layer.desc()
        K, N, r = layer.K, layer.N, layer.r
        act = layer.act
        self.X = torch.zeros((M, K), dtype=act, device=dev)
        self.dY = torch.zeros((M, N), dtype=act, device=dev)
        self.Y = torch.empty((M, N), dtype=act, device=dev)
        self.dX = torch.empty((M, K), dtype=act, device=dev)
        self.xA = torch.empty((M, r), dtype=torch.float32, device=dev)
        self.Xq = torch.empty((M, K), dtype=torch.int8, device=dev)
        self.sx = torch.empty((M,), dtype=torch.float32, device=dev)
        self.ws = qlora.workspace(self.desc, M, dev)
        # the trainable gradients in one flat buffer: dA [K,r], dB [r,N], dbias [N]
        self.grad_flat = torch.empty((K * r + r * N + N,), dtype=torch.float32, device=dev)
        self.dA = self.grad_flat[:K * r].view(K, r)
        self.dB = self.grad_flat[K * r:K * r + r * N].view(r, N)
        self.dbias = self.grad_flat[K * r + r * N:]
        self.graph: Optional[torch.cuda.CUDAGraph] = None
        # the X pass's stream and the fork/join events (None: one stream).  By
        # default from 512 tokens: below that the fork and join cost about as
        # much as the overlap saves (measured on the configurations' layers)
        if overlap_x is None:
            overlap_x = M >= 512
        self.side = torch.cuda.Stream(device=dev) if overlap_x else None
        self.fork = torch.cuda.Event() if overlap_x else None
        self.join = torch.cuda.Event() if overlap_x else None

    # ------------------------------------------------------------------
    def run(self, stream=None, events: Optional[Dict[str, Tuple[torch.cuda.Event, torch.cuda.Event]]] = None):
        L, D, M = self.layer, self.desc, self.M
        s = stream if stream is not None else torch.cuda.current_stream()

        def timed(name, fn, st=s):
            ev = events.get(name) if events else None
            if ev:
                ev[0].record(st)
            fn()
            if ev:
                ev[1].record(st)

        timed("quantize_input",
              lambda: qlora.qlora_quantize_input(D, M, self.X, L.A, self.Xq, self.sx, self.xA, s))
        timed("gemm_forward",
              lambda: qlora.qlora_gemm_forward(D, M, self.Xq, self.sx, L.Wq, L.sw, L.bias, self.xA,
                                               L.B, self.Y, None, s))
        timed("lora_grad_dy",
              lambda: qlora.qlora_lora_grad_dy(D, M, self.dY, L.B, self.xA, self.dB, self.dbias,
                                               self.ws, None, s))
        if self.side is None:
            timed("gemm_dx",
                  lambda: qlora.qlora_gemm_dx(D, M, self.dY, L.Wq, L.sw, L.A, self.dX, self.ws, s))
            timed("lora_grad_x", lambda: qlora.qlora_lora_grad_x(D, M, self.X, self.dA, self.ws, s))
            return
        # G is final: the X pass on the side stream, the dX GEMM here, then join
        # (the GEMM is issued first, at the library's greatest priority, so that
        # its CTAs take the SMs and the X pass runs in what they leave)
        x = self.side
        self.fork.record(s)
        timed("gemm_dx",
              lambda: qlora.qlora_gemm_dx(D, M, self.dY, L.Wq, L.sw, L.A, self.dX, self.ws, s))
        x.wait_event(self.fork)
        timed("lora_grad_x", lambda: qlora.qlora_lora_grad_x(D, M, self.X, self.dA, self.ws, x), x)
        self.join.record(x)
        s.wait_event(self.join)

    def make_events(self, parts=PARTS):
        return {p: (torch.cuda.Event(enable_timing=True, external=True),
                    torch.cuda.Event(enable_timing=True, external=True)) for p in parts}

    def capture(self, warmup: int = 1, events=None):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for _ in range(warmup):
                self.run()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.run(events=events)
        self.graph = g
        return g

    def replay(self):
        assert self.graph is not None
        self.graph.replay()

    # ------------------------------------------------------------------
    def launches_per_step(self) -> int:
        """Kernels this library launches in one step."""
        L = self.layer
        bf16 = L.act == torch.bfloat16
        rj = (L.r + 7) // 8
        dy_tc = bf16 and L.N % 8 == 0
        n = 2                                   # K1, K2
        n += 1 if dy_tc else rj                 # dY pass (G slices, dB, dbias)
        ncb = -(-L.N // 128) if dy_tc else -(-L.N // 64)
        n += 1 if ncb > 8 else 0                # G slices added once
        n += 1                                  # K3
        n += 1 if bf16 else rj                  # X pass
        return n

    def flops(self) -> float:
        """Algorithmic work of one step: int8 2MNK, the dX GEMM's 2MNK, and
        the rank-r products x.A, (xA).B, G = dY.B^T, G.A^T, dA, dB."""
        M, K, N, r = self.M, self.layer.K, self.layer.N, self.layer.r
        return 4.0 * M * N * K + 2.0 * M * r * (2 * K + 2 * N) + 2.0 * M * r * (K + N)


def algorithmic_bytes(M: int, K: int, N: int, r: int, e: int) -> Dict[str, float]:
    """Bytes each launch group must move at least once (e = activation bytes).

    quantize_input: X read, Xq/sx/xA written.  gemm_forward: Xq, Wq, Y, the
    scales, bias, xA, B.  lora_grad_dy: dY read, G, dB, dbias written, xA and
    B read.  gemm_dx: dY, Wq, dX, sw, G, A.  lora_grad_x: X, G, dA."""
    return {
        "quantize_input": M * K * e + M * K + 4.0 * M + 4.0 * M * r,
        "gemm_forward": M * K + K * N + M * N * e + 4.0 * (M + N + M * r + r * N + N),
        "lora_grad_dy": M * N * e + 4.0 * (M * r + r * N) + 4.0 * (M * r + r * N + N),
        "gemm_dx": M * N * e + K * N + M * K * e + 4.0 * (N + M * r + K * r),
        "lora_grad_x": M * K * e + 4.0 * (M * r + K * r),
    }
