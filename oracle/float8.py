"""CPU oracle of the float8 training recipe ("Introduce float8 training",
Keras PR 19488).  TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``:
imported by tests, smoke() and bench.py's CPU leg, never by the product.

What the page fixes: a Dense layer trained in float8 (quantization mode
"float8", QuantizedFloat8DTypePolicy), per-tensor scales and amax histories
("we can correctly update float8 parameters such as scale and
amax_history"; amax_history_length 1024 unless set), an output-gradient
scale (outputs_grad_scale), and float8 matmuls on float8 tensor cores.  It
prints no formula.  The readings this oracle takes (the plainest ones the
page supports; each is restated where it is used):

  * formats: inputs and kernel in E4M3 (4 exponent bits, bias 7, 3
    mantissa bits, no infinities, largest finite 448), the output gradient
    in E5M2 (5 exponent bits, bias 15, 2 mantissa bits, largest finite
    57344); subnormals included;
  * quantize: q = fp8(clip(fl32(t / s), -max, max)), the fp32 division
    rounded once, then round to nearest with ties to even on the format's
    grid (saturating: the clip keeps every value finite);
  * delayed scaling: a tensor is quantized with the scale stored by the
    previous step; the step then stores s' = fl32(h / max), h the largest
    entry of the amax history before this step's entry is added (s' = s
    when h is 0 or not finite), and the history becomes [amax, H[0], ..,
    H[L-2]] (this step's abs-max first, the oldest entry dropped);
  * the layer: Y = (Xq Wq) s_x s_w + bias;  dX = (dYq Wq^T) s_g s_w,
    dW = (Xq^T dYq) s_x s_g, dbias = column sums of dY (unquantized), the
    quantized tensors' products taken exactly (fp64 here).
"""
from __future__ import annotations

import numpy as np

E4M3 = "e4m3"
E5M2 = "e5m2"
MAX = {E4M3: 448.0, E5M2: 57344.0}
_BITS = {E4M3: (4, 3, 7), E5M2: (5, 2, 15)}  # exponent bits, mantissa bits, bias


def decode(codes, fmt):
    """uint8 codes -> float64 values (NaN for the NaN codes; E5M2's
    infinities as +-inf), from the format's definition."""
    e_bits, m_bits, bias = _BITS[fmt]
    c = np.asarray(codes, np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> m_bits) & ((1 << e_bits) - 1)
    m = c & ((1 << m_bits) - 1)
    sub = m.astype(np.float64) / (1 << m_bits) * 2.0 ** (1 - bias)
    nrm = (1.0 + m.astype(np.float64) / (1 << m_bits)) * 2.0 ** (e.astype(np.float64) - bias)
    v = sign * np.where(e == 0, sub, nrm)
    emax = (1 << e_bits) - 1
    if fmt == E4M3:
        v = np.where((e == emax) & (m == (1 << m_bits) - 1), np.nan, v)
    else:
        v = np.where((e == emax) & (m == 0), sign * np.inf, v)
        v = np.where((e == emax) & (m != 0), np.nan, v)
    return v


def _positive_grid(fmt):
    codes = np.arange(0x80, dtype=np.uint8)
    vals = decode(codes, fmt)
    keep = np.isfinite(vals) & (vals <= MAX[fmt])
    return codes[keep], vals[keep]


def encode(x, fmt):
    """float values (already within +-max) -> uint8 codes, round to nearest
    with ties to the even code (the one whose mantissa's last bit is 0)."""
    codes, vals = _positive_grid(fmt)  # ascending values, ascending codes
    x = np.asarray(x, np.float64)
    a = np.abs(x)
    if np.any(a > MAX[fmt]) or np.any(~np.isfinite(x)):
        raise ValueError("encode() takes finite values within +-max (clip first)")
    hi = np.clip(np.searchsorted(vals, a, side="left"), 0, len(vals) - 1)
    lo = np.clip(hi - 1, 0, len(vals) - 1)
    d_lo = np.abs(a - vals[lo])
    d_hi = np.abs(vals[hi] - a)
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (codes[hi] % 2 == 0) & (hi != lo))
    c = np.where(pick_hi, codes[hi], codes[lo]).astype(np.uint8)
    c = np.where(x < 0, c | 0x80, c).astype(np.uint8)
    # -0.0 and +0.0 both encode as 0x00
    return np.where(a == 0, np.uint8(0), c).astype(np.uint8)


def quantize(t, scale, fmt):
    """q = fp8(clip(fl32(t / s), -max, max)) as uint8 codes (t fp32 values)."""
    t32 = np.asarray(t, np.float32)
    v = (t32 / np.float32(scale)).astype(np.float32)
    v = np.clip(v, -MAX[fmt], MAX[fmt])
    return encode(v, fmt)


def next_scale(history, scale, fmt):
    """The scale stored for the next step: fl32(h / max), h = the largest
    history entry; the old scale when h is 0 or not finite."""
    h = np.float32(np.max(np.asarray(history, np.float32)))
    if not np.isfinite(h) or h <= 0:
        return np.float32(scale)
    return np.float32(h / np.float32(MAX[fmt]))


def next_history(history, amax):
    """[amax, H[0], .., H[L-2]]."""
    h = np.asarray(history, np.float32)
    return np.concatenate([[np.float32(amax)], h[:-1]]).astype(np.float32)


def step_tensor(t, state, fmt):
    """One step of one tensor: codes with the stored scale, then the new
    state.  state = dict(scale=float32, history=float32[L])."""
    t32 = np.asarray(t, np.float32)
    q = quantize(t32, state["scale"], fmt)
    amax = np.float32(np.max(np.abs(t32))) if t32.size else np.float32(0)
    new = {"scale": next_scale(state["history"], state["scale"], fmt),
           "history": next_history(state["history"], amax)}
    return q, amax, new


def forward(X, W, bias, sx, sw):
    """Y = (Xq Wq) s_x s_w + bias in fp64, X [M,K], W [K,N] (float values);
    returns dict(xq, wq, y)."""
    xq = quantize(X, sx, E4M3)
    wq = quantize(W, sw, E4M3)
    y = (decode(xq, E4M3) @ decode(wq, E4M3)) * (np.float64(sx) * np.float64(sw))
    if bias is not None:
        y = y + np.asarray(bias, np.float64)[None, :]
    return {"xq": xq, "wq": wq, "y": y}


def backward(X, W, dY, sx, sw, sg):
    """dX = (dYq Wq^T) s_g s_w, dW = (Xq^T dYq) s_x s_g, dbias = sum_m dY."""
    xq = decode(quantize(X, sx, E4M3), E4M3)
    wq = decode(quantize(W, sw, E4M3), E4M3)
    gq_codes = quantize(dY, sg, E5M2)
    gq = decode(gq_codes, E5M2)
    return {"gq": gq_codes,
            "dX": (gq @ wq.T) * (np.float64(sg) * np.float64(sw)),
            "dW": (xq.T @ gq) * (np.float64(sx) * np.float64(sg)),
            "dbias": np.asarray(dY, np.float64).sum(axis=0)}
