"""A Dense layer trained with the float8 recipe ("Introduce float8 training",
Keras PR 19488): the input and the kernel quantized to E4M3 and the output
gradient to E5M2 with per-tensor delayed scaling (a scale and an amax
history per tensor, updated every step), the three GEMMs of a training step
on float8 tensor cores.  The arithmetic runs in the library
(qlora_fp8_quantize[_colsum], qlora_fp8_gemm_ws, qlora_lora_grad_b for the
bias gradient where the quantizer cannot take it); this module only holds the state and orders the calls.

State per tensor: two device scales used in turn (a step quantizes with
one and writes the next into the other) and an amax history of
``history_len`` entries (1024 unless set, the page's default).  Scales start
at 1, histories at 0.
"""
from __future__ import annotations

from typing import Dict, Optional

import torch

from . import qlora


class Fp8State:
    """Delayed-scaling state of one tensor."""

    def __init__(self, history_len: int, device):
        self.scales = torch.ones(2, dtype=torch.float32, device=device)
        self.history = torch.zeros(history_len, dtype=torch.float32, device=device)
        self.cur = 0
        self.ws = torch.empty(qlora.FP8_WORKSPACE_BYTES, dtype=torch.uint8, device=device)
        self.cs_ws = None  # workspace of the quantization with column sums, grown on demand

    @property
    def scale(self) -> torch.Tensor:
        """The scale the next quantization uses (a one-element view)."""
        return self.scales[self.cur:self.cur + 1]

    def quantize(self, T: torch.Tensor, fmt: int, q: torch.Tensor, qt: Optional[torch.Tensor],
                 colsum: Optional[torch.Tensor] = None):
        """Codes of T (and, if colsum is given, T's column sums from the same
        pass); returns the scale they were made with (a view that stays valid
        until the state's second-next quantization)."""
        used = self.scales[self.cur:self.cur + 1]
        nxt = self.scales[1 - self.cur:2 - self.cur]
        if colsum is None:
            qlora.qlora_fp8_quantize(T, fmt, used, nxt, self.history, q, qt, self.ws)
        else:
            need = qlora.qlora_fp8_colsum_workspace_bytes(*T.shape)
            if self.cs_ws is None or self.cs_ws.numel() < need:
                self.cs_ws = torch.empty(need, dtype=torch.uint8, device=T.device)
            qlora.qlora_fp8_quantize_colsum(T, fmt, used, nxt, self.history, q, qt, colsum, self.cs_ws)
        self.cur = 1 - self.cur
        return used


class Float8Dense:
    """y = x W + b with float8 GEMMs; W [K, N] (fp32 master weights, trained),
    bias [N] or None; activations in `act` (bf16 or fp32)."""

    def __init__(self, W: torch.Tensor, bias: Optional[torch.Tensor] = None,
                 act: torch.dtype = torch.bfloat16, history_len: int = 1024):
        self.W = W.float().contiguous()
        self.K, self.N = self.W.shape
        self.bias = bias.float().contiguous() if bias is not None else None
        self.act = act
        dev = self.W.device
        self.sx = Fp8State(history_len, dev)
        self.sw = Fp8State(history_len, dev)
        self.sg = Fp8State(history_len, dev)
        self.gemm_ws = None  # the GEMMs' workspace (a split last wave of tiles), grown on demand
        self.Wq = torch.empty((self.K, self.N), dtype=torch.uint8, device=dev)   # for dX
        self.WqT = torch.empty((self.N, self.K), dtype=torch.uint8, device=dev)  # for Y

    def _gemm(self, A, fa, B, fb, sa, sb, bias, C):
        M, K = A.shape
        need = qlora.qlora_fp8_gemm_workspace_bytes(M, B.shape[0], K)
        if need and (self.gemm_ws is None or self.gemm_ws.numel() < need):
            self.gemm_ws = torch.empty(need, dtype=torch.uint8, device=A.device)
        qlora.qlora_fp8_gemm_ws(A, fa, B, fb, sa, sb, bias, C, self.gemm_ws if need else None)

    def forward(self, X: torch.Tensor) -> (torch.Tensor, Dict[str, torch.Tensor]):
        M = X.shape[0]
        dev = X.device
        Xq = torch.empty((M, self.K), dtype=torch.uint8, device=dev)
        XqT = torch.empty((self.K, M), dtype=torch.uint8, device=dev)
        s_x = self.sx.quantize(X, qlora.FP8_E4M3, Xq, XqT)
        s_w = self.sw.quantize(self.W, qlora.FP8_E4M3, self.Wq, self.WqT)
        Y = torch.empty((M, self.N), dtype=self.act, device=dev)
        self._gemm(Xq, qlora.FP8_E4M3, self.WqT, qlora.FP8_E4M3, s_x, s_w, self.bias, Y)
        return Y, {"Xq": Xq, "XqT": XqT, "s_x": s_x, "s_w": s_w}

    def backward(self, ctx: Dict[str, torch.Tensor], dY: torch.Tensor, want_dx: bool = True):
        """Returns dict(dX, dW, dbias, Gq)."""
        M = dY.shape[0]
        dev = dY.device
        Gq = torch.empty((M, self.N), dtype=torch.uint8, device=dev)
        GqT = torch.empty((self.N, M), dtype=torch.uint8, device=dev)
        # dbias = column sums of dY: from the quantizer's own pass where its
        # layout allows, else by the library's column-sum pass below
        fused = self.bias is not None and qlora.fp8_colsum_applies(dY, Gq, GqT)
        dbias = torch.empty((self.N,), dtype=torch.float32, device=dev) if fused else None
        s_g = self.sg.quantize(dY, qlora.FP8_E5M2, Gq, GqT, dbias)
        out = {"Gq": Gq, "s_g": s_g}
        if want_dx:
            dX = torch.empty((M, self.K), dtype=self.act, device=dev)
            self._gemm(Gq, qlora.FP8_E5M2, self.Wq, qlora.FP8_E4M3, s_g, ctx["s_w"], None, dX)
            out["dX"] = dX
        dW = torch.empty((self.K, self.N), dtype=torch.float32, device=dev)
        self._gemm(ctx["XqT"], qlora.FP8_E4M3, GqT, qlora.FP8_E5M2, ctx["s_x"], s_g, None, dW)
        out["dW"] = dW
        if fused:
            out["dbias"] = dbias
        elif self.bias is not None:
            # column sums of dY by the library's pass (its dB output, for a
            # rank-1 factor of zeros, is discarded)
            d = qlora.desc(16, self.N, 1, 1.0, dY.dtype)
            zeros = torch.zeros((M, 1), dtype=torch.float32, device=dev)
            scratch = torch.empty((1, self.N), dtype=torch.float32, device=dev)
            dbias = torch.empty((self.N,), dtype=torch.float32, device=dev)
            qlora.qlora_lora_grad_b(d, M, dY, zeros, scratch, dbias)
            out["dbias"] = dbias
        return out
