"""EinsumDense equations on the int8-LoRA Dense layer.

Keras' EinsumDense ("Introduce QLoRA-like technique", Results table: the
EinsumDense rows; "Introduce float8 training" and the GPT-2 LoRA notebook use
it for the attention projections) writes a projection as an einsum, e.g.
"btd,dnh->btnh" (query/key/value: model width d into n heads of width h) or
"btnh,nhd->btd" (attention output).  When the equation contracts the
trailing axes of the input with the leading axes of the kernel and keeps the
remaining axes in order (input's first, then kernel's), it is the Dense layer
on the flattened axes:

    X [prod(batch), K = prod(contracted)] x W [K, N = prod(free)]

so the int8 kernels run unchanged on contiguous reshapes; nothing is copied.
The LoRA factors follow the same flattening: A [contracted..., r] is
A [K, r] and B [r, free...] is B [r, N].  keras-llm-light keeps a per-head
B [heads, r, head_dim] for the query projection (its block summary:
query/lora_B [8, 4, 256]); ``b_per_head()`` gives that layout as a strided
view of the Dense B.  Other equations (a contraction axis in the middle of
the input, permuted outputs) raise ValueError.
"""
from __future__ import annotations

from dataclasses import dataclass
from math import prod
from typing import Dict, List, Tuple

import torch

from . import qlora


@dataclass(frozen=True)
class EinsumPlan:
    equation: str
    batch: str       # input axes kept in the output (leading)
    contracted: str  # input trailing axes = kernel leading axes
    free: str        # kernel trailing axes (trailing in the output)


def plan(equation: str) -> EinsumPlan:
    """Checks that `equation` is a Dense layer on flattened axes and splits
    its axes into batch, contracted and free ones."""
    eq = equation.replace(" ", "")
    try:
        lhs, out = eq.split("->")
        x, w = lhs.split(",")
    except ValueError:
        raise ValueError("expected an equation 'input,kernel->output', got %r" % equation)
    for part in (x, w, out):
        if not part.isalpha() or len(set(part)) != len(part):
            raise ValueError("axes must be distinct letters: %r" % equation)
    contracted = "".join(c for c in x if c in w and c not in out)
    n = len(contracted)
    if n == 0 or x[len(x) - n:] != contracted or w[:n] != contracted:
        raise ValueError("%r: the contracted axes must be the trailing input axes and the leading "
                         "kernel axes, in the same order" % equation)
    batch, free = x[:len(x) - n], w[n:]
    if out != batch + free:
        raise ValueError("%r: the output must be the input's kept axes followed by the kernel's "
                         "free axes, %r" % (equation, batch + free))
    if set(batch) & set(free):
        raise ValueError("%r: an axis of the input and of the kernel share a letter" % equation)
    return EinsumPlan(eq, batch, contracted, free)


def flat_shapes(p: EinsumPlan, x_shape, w_shape):
    """(M, K, N, batch_shape, contracted_shape, free_shape) of the Dense
    layer that equation plan `p` is, for an input of shape `x_shape` and a
    kernel of shape `w_shape`.  The flattened operands are plain reshapes
    (row-major) of the einsum ones: X [M, K], W [K, N], A [K, r], B [r, N]."""
    nb, nc = len(p.batch), len(p.contracted)
    if len(x_shape) != nb + nc or len(w_shape) != nc + len(p.free):
        raise ValueError("operand ranks do not match %r" % p.equation)
    contracted = tuple(w_shape[:nc])
    if tuple(x_shape[nb:]) != contracted:
        raise ValueError("input axes %s do not match the kernel's %s" % (tuple(x_shape[nb:]), contracted))
    batch, free = tuple(x_shape[:nb]), tuple(w_shape[nc:])
    return prod(batch), prod(contracted), prod(free), batch, contracted, free


class EinsumDense:
    """An int8-LoRA EinsumDense layer: frozen int8 kernel, fp32 LoRA factors.

    kernel: the float kernel in the equation's layout (contracted..., free...).
    """

    def __init__(self, equation: str, kernel: torch.Tensor, rank: int, alpha: float,
                 act: torch.dtype = torch.bfloat16, bias: torch.Tensor = None,
                 A: torch.Tensor = None, B: torch.Tensor = None):
        self.plan = plan(equation)
        p = self.plan
        if kernel.dim() != len(p.contracted) + len(p.free):
            raise ValueError("kernel has %d axes, the equation %d" %
                             (kernel.dim(), len(p.contracted) + len(p.free)))
        self.contracted_shape = tuple(kernel.shape[:len(p.contracted)])
        self.free_shape = tuple(kernel.shape[len(p.contracted):])
        self.K = prod(self.contracted_shape)
        self.N = prod(self.free_shape)
        if bias is not None:
            bias = bias.reshape(self.N).float().contiguous()
        dev = kernel.device
        Wq, sw = qlora.quantize_weight(kernel.reshape(self.K, self.N).float().contiguous())
        if A is None:
            A = torch.zeros((self.K, rank), dtype=torch.float32, device=dev)
        if B is None:
            B = torch.zeros((rank, self.N), dtype=torch.float32, device=dev)
        self.layer = qlora.Layer(Wq=Wq, sw=sw, bias=bias,
                                 A=A.reshape(self.K, rank).float().contiguous(),
                                 B=B.reshape(rank, self.N).float().contiguous(),
                                 alpha=alpha, act=act)
        self.r = rank

    # ---------------------------------------------------------------- layouts
    def _flat_x(self, X: torch.Tensor) -> Tuple[torch.Tensor, Tuple[int, ...]]:
        M, _, _, batch_shape, _, _ = flat_shapes(self.plan, tuple(X.shape),
                                                 self.contracted_shape + self.free_shape)
        if not X.is_contiguous():
            raise ValueError("the input must be contiguous (the axes are flattened in place)")
        return X.view(M, self.K), batch_shape

    def a_view(self) -> torch.Tensor:
        """A in the equation's layout: [contracted..., r]."""
        return self.layer.A.view(*self.contracted_shape, self.r)

    def b_view(self) -> torch.Tensor:
        """B in the equation's layout: [r, free...]."""
        return self.layer.B.view(self.r, *self.free_shape)

    def b_per_head(self) -> torch.Tensor:
        """B as [free[0], r, free[1:]...] (per-head factors, e.g. [heads, r,
        head_dim]); a strided view of the same storage, no copy."""
        if len(self.free_shape) < 2:
            raise ValueError("a per-head view needs at least two free axes")
        return self.b_view().transpose(0, 1)

    # ---------------------------------------------------------------- compute
    def workspace(self, X: torch.Tensor) -> torch.Tensor:
        Xf, _ = self._flat_x(X)
        return qlora.workspace(self.layer.desc(), Xf.shape[0], X.device)

    def forward(self, X: torch.Tensor, ws: torch.Tensor):
        """Returns (Y [batch..., free...], xA [prod(batch), r])."""
        Xf, batch_shape = self._flat_x(X)
        Y, xA = qlora.forward(self.layer, Xf, ws)
        return Y.view(*batch_shape, *self.free_shape), xA

    def backward(self, X: torch.Tensor, dY: torch.Tensor, xA: torch.Tensor, ws: torch.Tensor,
                 want_dx: bool = True) -> Dict[str, torch.Tensor]:
        """Returns dX in the input's layout, dA [contracted..., r], dB [r,
        free...] and dbias [free...] (views of the flat results)."""
        Xf, batch_shape = self._flat_x(X)
        if not dY.is_contiguous() or tuple(dY.shape) != batch_shape + self.free_shape:
            raise ValueError("dY must be a contiguous %s tensor" % (batch_shape + self.free_shape,))
        dX, dA, dB, dbias = qlora.backward(self.layer, Xf, dY.view(Xf.shape[0], self.N), xA, ws,
                                           want_dx=want_dx)
        return {"dX": dX.view(X.shape) if dX is not None else None,
                "dA": dA.view(*self.contracted_shape, self.r),
                "dB": dB.view(self.r, *self.free_shape),
                "dbias": dbias.view(*self.free_shape) if dbias is not None else None}


def supported(equation: str) -> bool:
    try:
        plan(equation)
        return True
    except ValueError:
        return False


__all__: List[str] = ["EinsumDense", "EinsumPlan", "flat_shapes", "plan", "supported"]
