"""The MNIST MLP workload as a stack of int8-LoRA Dense layers on one GPU.

784 -> 1024, 31 x (1024 -> 1024), 1024 -> 10 with a ReLU between layers
("Introduce QLoRA-like technique", benchmark.py and its Results table),
batch 1024, bf16 activations, rank-8 adapters.  One ``step`` is the forward
through every layer and the backward through every layer (dX, dA, dB of
each), all through the C ABI into preallocated device buffers, so a step can
be captured into a CUDA graph and replayed.  The ReLU runs in the epilogues:
the forward GEMM of a hidden layer writes max(Y, 0), and the dX GEMM of a
layer whose input came out of a ReLU zeroes dX where that input is <= 0.
"""
from __future__ import annotations

from typing import Dict, List, Optional

import torch

from . import inputs as _inputs
from . import qlora


class MLPStack:
    # rows per CTA of the dB/dbias and dA passes on the side stream
    SIDE_PASS_ROWS = 256

    def __init__(self, layers: List[qlora.Layer], batch: int, device="cuda"):
        self.layers = layers
        self.M = batch
        self.act = layers[0].act
        dev = torch.device(device)
        # the largest workspace over the layers serves all of them; two of them
        # alternate between layers in the backward, so that a layer's X pass
        # (on the side stream) can still read its G while the next layer's
        # dY pass writes the other one
        need = max(qlora.qlora_workspace_bytes(L.desc(), batch) for L in layers)
        self.ws = torch.empty(need, dtype=torch.uint8, device=dev)
        self.ws_alt = torch.empty(need, dtype=torch.uint8, device=dev)
        # only G feeds the next layer's gradient: the G pass and the dX GEMM
        # carry the critical path, while each layer's dB/dbias pass and X pass
        # (dA) run on a side stream, overlapping the next layers
        self.side = torch.cuda.Stream(device=dev)
        self.ev_g = [torch.cuda.Event() for _ in layers]  # layer's G is in its workspace
        self.ev_x = [torch.cuda.Event() for _ in layers]  # layer's X pass is done
        self.ev_dx = [torch.cuda.Event() for _ in layers]  # layer's dX GEMM is done (timed layers)
        self.X = torch.zeros((batch, layers[0].K), dtype=self.act, device=dev)
        self.dY = torch.zeros((batch, layers[-1].N), dtype=self.act, device=dev)
        self.H = [torch.empty((batch, L.N), dtype=self.act, device=dev) for L in layers]
        self.xA = [torch.empty((batch, L.r), dtype=torch.float32, device=dev) for L in layers]
        self.G = [torch.empty((batch, L.N), dtype=self.act, device=dev) for L in layers]
        self.dX = torch.empty((batch, layers[0].K), dtype=self.act, device=dev)
        self.dbias = [torch.empty((L.N,), dtype=torch.float32, device=dev) for L in layers]
        Kmax = max(L.K for L in layers)
        self.Xq = torch.empty((batch, Kmax), dtype=torch.int8, device=dev)
        self.sx = torch.empty((batch,), dtype=torch.float32, device=dev)
        # the LoRA gradients live in one flat buffer (one all-reduce in data
        # parallel runs); dA[i], dB[i] are views into it
        sizes = [L.K * L.r + L.r * L.N for L in layers]
        self.grad_flat = torch.empty((sum(sizes),), dtype=torch.float32, device=dev)
        off = 0
        self.dA, self.dB = [], []
        for L in layers:
            self.dA.append(self.grad_flat[off:off + L.K * L.r].view(L.K, L.r))
            off += L.K * L.r
            self.dB.append(self.grad_flat[off:off + L.r * L.N].view(L.r, L.N))
            off += L.r * L.N
        self.descs = [L.desc() for L in layers]
        self.graph: Optional[torch.cuda.CUDAGraph] = None
        self.events = None

    @classmethod
    def from_inputs(cls, specs: List[_inputs.LayerSpec], data: Dict[str, object], device="cuda"):
        layers = []
        act = torch.bfloat16 if specs[0].act == "bf16" else torch.float32
        for s, L in zip(specs, data["layers"]):
            Wq, sw = qlora.quantize_weight(torch.from_numpy(L["W"]).to(device))
            bias = torch.from_numpy(L["bias"]).to(device) if L["bias"] is not None else None
            layers.append(qlora.Layer(Wq=Wq, sw=sw, bias=bias,
                                      A=torch.from_numpy(L["A"]).to(device),
                                      B=torch.from_numpy(L["B"]).to(device),
                                      alpha=s.alpha, act=act))
        return cls(layers, specs[0].M, device)

    # ------------------------------------------------------------------
    def launches_per_step(self) -> int:
        """Kernels this library launches in one step (for the benchmark)."""
        n = 0
        bf16 = self.act == torch.bfloat16
        for i, L in enumerate(self.layers):
            n += 2                                   # quantize+xA, int8 GEMM (+ ReLU)
            rj = (L.r + 7) // 8                      # CUDA-core passes: 8 ranks per launch
            dy_tc = bf16 and L.N % 8 == 0            # tensor-core dY passes, 128-column blocks
            n += 2 if dy_tc else 2 * rj              # G pass + dB/dbias pass
            ncb = -(-L.N // 128) if dy_tc else -(-L.N // 64)
            n += 1 if ncb > 8 else 0                 # G slices added once
            n += 1                                   # dX GEMM (+ ReLU backward)
            n += 1 if bf16 else rj                   # X pass
        return n

    def _run(self, stream=None, events=None):
        """One step.  ``events`` optionally maps a step name ("gemm_forward"
        or "gemm_dx") to a per-layer list of (start, end) CUDA events, or
        None for a layer that is not timed, recorded around that launch."""
        L_ = self.layers
        n = len(L_)
        D = self.descs
        M = self.M
        ev_f = events.get("gemm_forward") if events else None
        fwd = stream if stream is not None else torch.cuda.current_stream()
        ev_d = events.get("gemm_dx") if events else None
        h = self.X
        for i, L in enumerate(L_):
            qlora.qlora_quantize_input(D[i], M, h, L.A, self.Xq, self.sx, self.xA[i], stream)
            if ev_f and ev_f[i]:
                ev_f[i][0].record(fwd)
            # hidden layers: the ReLU that follows runs in the GEMM's epilogue
            gemm = qlora.qlora_gemm_forward_relu if i < n - 1 else qlora.qlora_gemm_forward
            gemm(D[i], M, self.Xq, self.sx, L.Wq, L.sw, L.bias, self.xA[i], L.B, self.H[i], None,
                 stream)
            if ev_f and ev_f[i]:
                ev_f[i][1].record(fwd)
            h = self.H[i]
        main = stream if stream is not None else torch.cuda.current_stream()
        # the side-stream passes cover 256 rows per CTA: half the CTAs of the
        # default spread, so that they leave the SMs to the dX GEMMs
        prev = qlora.qlora_set_rank_pass_rows(self.SIDE_PASS_ROWS)
        try:
            self._backward(main, ev_d)
        finally:
            qlora.qlora_set_rank_pass_rows(prev)

    def _backward(self, main, ev_d):
        L_ = self.layers
        n = len(L_)
        D = self.descs
        M = self.M
        g = self.dY
        for i in range(n - 1, -1, -1):
            L = L_[i]
            ws = self.ws if i % 2 == 0 else self.ws_alt
            x_in = self.X if i == 0 else self.H[i - 1]
            dX = self.dX if i == 0 else self.G[i - 1]
            if i + 2 < n:
                main.wait_event(self.ev_x[i + 2])  # the X pass that read this workspace
            qlora.qlora_lora_g(D[i], M, g, L.B, ws, main)
            self.ev_g[i].record(main)
            if ev_d and ev_d[i]:
                ev_d[i][0].record(main)
            if i > 0:
                # dX taken back through the ReLU that produced this layer's input
                qlora.qlora_gemm_dx_relu(D[i], M, g, L.Wq, L.sw, L.A, x_in, dX, ws, main)
            else:
                qlora.qlora_gemm_dx(D[i], M, g, L.Wq, L.sw, L.A, dX, ws, main)
            if ev_d and ev_d[i]:
                ev_d[i][1].record(main)
                self.ev_dx[i].record(main)
            # a timed dX GEMM runs alone: the side stream waits until it ends
            # (through an ordinary event: a timing event cannot carry a stream
            # into a graph capture)
            self.side.wait_event(self.ev_dx[i] if ev_d and ev_d[i] else self.ev_g[i])
            qlora.qlora_lora_grad_b(D[i], M, g, self.xA[i], self.dB[i], self.dbias[i], self.side)
            qlora.qlora_lora_grad_x(D[i], M, x_in, self.dA[i], ws, self.side)
            self.ev_x[i].record(self.side)
            g = dX
        main.wait_stream(self.side)

    def make_events(self, kinds=("gemm_dx",), layers=None):
        """Timing events (graph-capturable) around the given steps of the
        given layers (all layers when None).  An event pair between two
        kernels orders them, so each timed launch loses its overlap with its
        neighbours, and a timed dX GEMM also keeps that layer's side-stream
        passes waiting until it ends; time a few layers to keep the step
        itself close to unperturbed."""
        sel = set(range(len(self.layers)) if layers is None else layers)
        return {k: [(torch.cuda.Event(enable_timing=True, external=True),
                     torch.cuda.Event(enable_timing=True, external=True)) if i in sel else None
                    for i in range(len(self.layers))] for k in kinds}

    def capture(self, warmup: int = 1, events=None):
        """Records one step into a CUDA graph (after `warmup` eager steps)."""
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for _ in range(warmup):
                self._run()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self._run(events=events)
        self.graph = g
        self.events = events
        return g

    def replay(self):
        assert self.graph is not None
        self.graph.replay()

    def step(self, X: Optional[torch.Tensor] = None, dY: Optional[torch.Tensor] = None,
             use_graph: bool = False):
        if X is not None:
            self.X.copy_(X)
        if dY is not None:
            self.dY.copy_(dY)
        if use_graph:
            self.replay()
        else:
            self._run()
        return {"y": self.H[-1], "dX": self.dX, "dA": self.dA, "dB": self.dB, "dbias": self.dbias}

    # ------------------------------------------------------------------
    def flops_per_step(self) -> float:
        """Algorithmic work of one step: int8 2MNK + bf16 2MNK per layer plus
        the rank-r terms (x.A, (xA).B, G, G.A^T, dA, dB)."""
        tot = 0.0
        M = self.M
        for L in self.layers:
            tot += 2.0 * M * L.N * L.K * 2
            tot += 2.0 * M * L.r * (2 * L.K + 2 * L.N) + 2.0 * M * L.r * (L.K + L.N)
        return tot
