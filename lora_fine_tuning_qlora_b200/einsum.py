"""EinsumDense equations on the int8-LoRA Dense layer.

Keras' EinsumDense ("Introduce QLoRA-like technique", Results table: the
EinsumDense rows; "Introduce float8 training": "ab,bcd->acd" and the speed
test's "abcde,aebf->adbcf"; the GPT-2 LoRA notebook's attention projections)
writes a projection as an einsum of an input and a kernel.  Its axes fall
into four groups:

  batch       in the input, the kernel and the output (one kernel slice each)
  kept        in the input and the output
  contracted  in the input and the kernel, summed over
  free        in the kernel and the output

so the equation is, for every batch index, the Dense layer

    X_b [prod(kept), K = prod(contracted)] x W_b [K, N = prod(free)]

on operands brought to [batch, kept, contracted] (input), [batch,
contracted, free] (kernel) and [batch, kept, free] (output) order.  When
there is no batch axis and the operands already are in that order (e.g.
"btd,dnh->btnh", "btnh,nhd->btd"), the layer runs on reshapes and nothing is
copied; otherwise the library's permutation kernel moves the input, the
upstream gradient and the results between the equation's order and the
layer's (qlora_permute).  The int8 kernel of each batch slice is quantized
per output channel of that slice.

The LoRA factors follow the notebook's construction (its lora_A contracts
the same input axes as the kernel down to the rank, its lora_B maps the rank
to the kernel's free axes): A [contracted..., r] and B [r, free...], one pair
per batch slice when the equation has batch axes (A [batch..., contracted...,
r], B [batch..., r, free...]).  keras-llm-light keeps a per-head B [heads, r,
head_dim] for the query projection; ``b_per_head()`` gives that layout as a
strided view.  The bias, if any, has the free axes' shape and is shared by
the batch slices.  Equations that sum an axis of one operand only, or repeat
a letter, raise ValueError.
"""
from __future__ import annotations

from dataclasses import dataclass
from math import prod
from typing import Dict, List, Optional, Tuple

import torch

from . import qlora


@dataclass(frozen=True)
class EinsumPlan:
    equation: str
    x: str
    w: str
    out: str
    batch: str       # axes of all three operands, in output order
    kept: str        # input and output axes, in output order
    contracted: str  # input and kernel axes, in input order
    free: str        # kernel and output axes, in output order

    @property
    def x_perm(self) -> Tuple[int, ...]:
        """Input axes in [batch, kept, contracted] order."""
        return tuple(self.x.index(c) for c in self.batch + self.kept + self.contracted)

    @property
    def w_perm(self) -> Tuple[int, ...]:
        """Kernel axes in [batch, contracted, free] order."""
        return tuple(self.w.index(c) for c in self.batch + self.contracted + self.free)

    @property
    def out_perm(self) -> Tuple[int, ...]:
        """[batch, kept, free] axes in the output's order."""
        canon = self.batch + self.kept + self.free
        return tuple(canon.index(c) for c in self.out)

    @property
    def flat(self) -> bool:
        """A Dense layer on plain reshapes: no batch axis, no permutation."""
        ident = lambda p: tuple(p) == tuple(range(len(p)))
        return not self.batch and ident(self.x_perm) and ident(self.w_perm) and ident(self.out_perm)


def plan(equation: str) -> EinsumPlan:
    """Splits the axes of 'input,kernel->output' into batch, kept,
    contracted and free groups; raises ValueError for equations that are not
    a (batched) Dense layer."""
    eq = equation.replace(" ", "")
    try:
        lhs, out = eq.split("->")
        x, w = lhs.split(",")
    except ValueError:
        raise ValueError("expected an equation 'input,kernel->output', got %r" % equation)
    for part in (x, w, out):
        if not part.isalpha() or len(set(part)) != len(part):
            raise ValueError("axes must be distinct letters: %r" % equation)
    for c in x:
        if c not in w and c not in out:
            raise ValueError("%r: input axis %r is summed over without the kernel" % (equation, c))
    for c in w:
        if c not in x and c not in out:
            raise ValueError("%r: kernel axis %r is summed over without the input" % (equation, c))
    for c in out:
        if c not in x and c not in w:
            raise ValueError("%r: output axis %r is in neither operand" % (equation, c))
    batch = "".join(c for c in out if c in x and c in w)
    kept = "".join(c for c in out if c in x and c not in w)
    free = "".join(c for c in out if c in w and c not in x)
    contracted = "".join(c for c in x if c in w and c not in out)
    if not contracted:
        raise ValueError("%r: no contracted axis" % equation)
    return EinsumPlan(eq, x, w, out, batch, kept, contracted, free)


def flat_shapes(p: EinsumPlan, x_shape, w_shape):
    """(nb, M, K, N, sizes) of plan `p` for an input of shape `x_shape` and a
    kernel of shape `w_shape`: nb batch slices of a Dense layer with M =
    prod(kept), K = prod(contracted), N = prod(free); sizes maps every axis
    letter to its extent."""
    if len(x_shape) != len(p.x) or len(w_shape) != len(p.w):
        raise ValueError("operand ranks do not match %r" % p.equation)
    sizes: Dict[str, int] = {}
    for letters, shape in ((p.x, x_shape), (p.w, w_shape)):
        for c, n in zip(letters, shape):
            if sizes.setdefault(c, int(n)) != int(n):
                raise ValueError("axis %r has extents %d and %d" % (c, sizes[c], n))
    ext = lambda s: prod(sizes[c] for c in s)
    return ext(p.batch), ext(p.kept), ext(p.contracted), ext(p.free), sizes


def _permute(t: torch.Tensor, perm) -> torch.Tensor:
    if tuple(perm) == tuple(range(t.dim())):
        return t.contiguous()
    return qlora.qlora_permute(t.contiguous(), perm)


def _inverse(perm) -> Tuple[int, ...]:
    inv = [0] * len(perm)
    for d, p in enumerate(perm):
        inv[p] = d
    return tuple(inv)


class EinsumDense:
    """An int8-LoRA EinsumDense layer: frozen int8 kernel, fp32 LoRA factors.

    kernel: the float kernel in the equation's layout.  A, B (optional, zeros
    by default): [batch..., contracted..., r] and [batch..., r, free...]
    (without the batch axes when the equation has none).
    """

    def __init__(self, equation: str, kernel: torch.Tensor, rank: int, alpha: float,
                 act: torch.dtype = torch.bfloat16, bias: Optional[torch.Tensor] = None,
                 A: Optional[torch.Tensor] = None, B: Optional[torch.Tensor] = None):
        self.plan = p = plan(equation)
        if kernel.dim() != len(p.w):
            raise ValueError("kernel has %d axes, the equation %d" % (kernel.dim(), len(p.w)))
        self.w_sizes = {c: int(n) for c, n in zip(p.w, kernel.shape)}
        ext = lambda s: prod(self.w_sizes[c] for c in s)
        self.batch_shape = tuple(self.w_sizes[c] for c in p.batch)
        self.contracted_shape = tuple(self.w_sizes[c] for c in p.contracted)
        self.free_shape = tuple(self.w_sizes[c] for c in p.free)
        self.nb, self.K, self.N = ext(p.batch), ext(p.contracted), ext(p.free)
        self.r = rank
        self.alpha = alpha
        self.act = act
        dev = kernel.device
        Wc = _permute(kernel.float(), p.w_perm).view(self.nb, self.K, self.N)
        self.Wq = torch.empty((self.nb, self.N, self.K), dtype=torch.int8, device=dev)
        self.sw = torch.empty((self.nb, self.N), dtype=torch.float32, device=dev)
        for b in range(self.nb):
            qlora.qlora_quantize_weight(Wc[b], self.Wq[b], self.sw[b])
        self.bias = bias.reshape(self.N).float().contiguous() if bias is not None else None
        self.A = (A.reshape(self.nb, self.K, rank).float().contiguous() if A is not None
                  else torch.zeros((self.nb, self.K, rank), dtype=torch.float32, device=dev))
        self.B = (B.reshape(self.nb, rank, self.N).float().contiguous() if B is not None
                  else torch.zeros((self.nb, rank, self.N), dtype=torch.float32, device=dev))
        self.layers = [qlora.Layer(Wq=self.Wq[b], sw=self.sw[b], bias=self.bias, A=self.A[b],
                                   B=self.B[b], alpha=alpha, act=act) for b in range(self.nb)]

    # ---------------------------------------------------------------- layouts
    @property
    def layer(self) -> qlora.Layer:
        """The Dense layer of an equation without batch axes."""
        if self.nb != 1 or self.plan.batch:
            raise ValueError("the equation has batch axes: one layer per slice (self.layers)")
        return self.layers[0]

    def _shapes(self, X: torch.Tensor):
        nb, M, K, N, sizes = flat_shapes(self.plan, tuple(X.shape),
                                         tuple(self.w_sizes[c] for c in self.plan.w))
        return M, sizes

    def _canon_x(self, X: torch.Tensor) -> torch.Tensor:
        M, _ = self._shapes(X)
        if self.plan.flat:
            if not X.is_contiguous():
                raise ValueError("the input must be contiguous (the axes are flattened in place)")
            return X.view(1, M, self.K)
        return _permute(X, self.plan.x_perm).view(self.nb, M, self.K)

    def _out_shape(self, sizes, letters) -> Tuple[int, ...]:
        return tuple(sizes[c] for c in letters)

    def a_view(self) -> torch.Tensor:
        """A in the equation's layout: [batch..., contracted..., r]."""
        return self.A.view(*self.batch_shape, *self.contracted_shape, self.r)

    def b_view(self) -> torch.Tensor:
        """B in the equation's layout: [batch..., r, free...]."""
        return self.B.view(*self.batch_shape, self.r, *self.free_shape)

    def b_per_head(self) -> torch.Tensor:
        """B as [free[0], r, free[1:]...] (per-head factors, e.g. [heads, r,
        head_dim]); a strided view of the same storage, no copy."""
        if self.plan.batch:
            raise ValueError("per-head factors are defined for equations without batch axes")
        if len(self.free_shape) < 2:
            raise ValueError("a per-head view needs at least two free axes")
        return self.b_view().transpose(0, 1)

    # ---------------------------------------------------------------- compute
    def workspace(self, X: torch.Tensor) -> torch.Tensor:
        M, _ = self._shapes(X)
        return qlora.workspace(self.layers[0].desc(), M, X.device)

    def forward(self, X: torch.Tensor, ws: torch.Tensor):
        """Returns (Y in the equation's output layout, xA [nb, M, r]).  For an
        equation without batch axes xA is [M, r]."""
        M, sizes = self._shapes(X)
        Xc = self._canon_x(X)
        p = self.plan
        Yc = torch.empty((self.nb, M, self.N), dtype=self.act, device=X.device)
        xA = torch.empty((self.nb, M, self.r), dtype=torch.float32, device=X.device)
        for b, L in enumerate(self.layers):
            qlora.forward(L, Xc[b], ws, Y=Yc[b], xA=xA[b])
        canon = self._out_shape(sizes, p.batch + p.kept + p.free)
        Y = Yc.view(canon) if p.flat else _permute(Yc.view(canon), p.out_perm)
        return Y, (xA[0] if not p.batch else xA)

    def backward(self, X: torch.Tensor, dY: torch.Tensor, xA: torch.Tensor, ws: torch.Tensor,
                 want_dx: bool = True) -> Dict[str, torch.Tensor]:
        """Returns dX in the input's layout, dA [batch..., contracted..., r],
        dB [batch..., r, free...] and dbias [free...] (summed over the batch
        slices)."""
        M, sizes = self._shapes(X)
        p = self.plan
        if tuple(dY.shape) != self._out_shape(sizes, p.out):
            raise ValueError("dY must have the output's shape %s" % (self._out_shape(sizes, p.out),))
        Xc = self._canon_x(X)
        if p.flat:
            if not dY.is_contiguous():
                raise ValueError("dY must be contiguous")
            dYc = dY.view(1, M, self.N)
        else:
            dYc = _permute(dY, _inverse(p.out_perm)).view(self.nb, M, self.N)
        xAb = xA.view(self.nb, M, self.r)
        dXc = torch.empty((self.nb, M, self.K), dtype=self.act, device=X.device) if want_dx else None
        dA = torch.empty((self.nb, self.K, self.r), dtype=torch.float32, device=X.device)
        dB = torch.empty((self.nb, self.r, self.N), dtype=torch.float32, device=X.device)
        dbias = torch.empty((self.N,), dtype=torch.float32, device=X.device)
        for b, L in enumerate(self.layers):
            qlora.qlora_backward(L.desc(), M, Xc[b], dYc[b], L.Wq, L.sw, L.A, L.B, xAb[b],
                                 dXc[b] if want_dx else None, dA[b], dB[b],
                                 dbias if self.nb == 1 else None, ws)
        if self.nb > 1:
            # the shared bias: column sums of dY over every slice's rows (the
            # dB of that call, over all slices at once, is not used)
            scratch = torch.empty((self.r, self.N), dtype=torch.float32, device=X.device)
            qlora.qlora_lora_grad_b(self.layers[0].desc(), self.nb * M, dYc.view(self.nb * M, self.N),
                                    xAb.reshape(self.nb * M, self.r), scratch, dbias)
        dX = None
        if want_dx:
            canon_x = self._out_shape(sizes, p.batch + p.kept + p.contracted)
            dX = (dXc.view(X.shape) if p.flat
                  else _permute(dXc.view(canon_x), _inverse(p.x_perm)))
        return {"dX": dX,
                "dA": dA.view(*self.batch_shape, *self.contracted_shape, self.r),
                "dB": dB.view(*self.batch_shape, self.r, *self.free_shape),
                "dbias": dbias.view(*self.free_shape)}


def supported(equation: str) -> bool:
    try:
        plan(equation)
        return True
    except ValueError:
        return False


__all__: List[str] = ["EinsumDense", "EinsumPlan", "flat_shapes", "plan", "supported"]
