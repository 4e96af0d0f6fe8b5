"""CPU oracle for the int8-frozen-kernel LoRA Dense layer.

TEST INFRASTRUCTURE ONLY.  This package is imported by ``tests/``, by
``__graft_entry__.smoke()`` and by the CPU-baseline leg of ``bench.py``; the
product path (``lora_fine_tuning_qlora_b200``) never imports, links or calls
it, and it never imports the product.  The arithmetic lives in the plain C
file ``qlora_oracle.c`` next to this module (scalar loops, fp64 sums, fp32
quantization); this module only marshals numpy arrays into it, plus the
composition of layers into the MLP stack workload (a plain ReLU between
layers).

What each routine follows (page title, section):
  * quantize_weight / quantize_rows -- "Introduce QLoRA-like technique"
    (Keras PR 19356), Highlights: frozen int8 kernel; the quantizer itself
    (symmetric abs-max, scale amax/127, round half to even, fp32) is the
    reading stated in the C file's header, since the pages give no formula.
  * int8_matmul / forward -- same page, Results (int8 Dense); "Parameter-
    efficient fine-tuning of GPT-2 with LoRA", "LoRA equation" and "Create
    LoRA layer" (scale alpha / rank).
  * backward -- gradients reach only the LoRA factors, the int8 kernel is
    frozen ("How to fine-tune the 4-bit model?" thread); straight-through
    through the input quantizer.
  * merge -- Keras PR 19356 Results footnote (lossy merge) and the 4-bit
    thread (de-quantize, add the LoRA, re-quantize).
  * quantize_outlier_int8 / dequantize_outlier_int8 / percentile / round_fp16
    -- outlier-compensated int8 kernels: keras-llm-light, "Weights
    quantization" and "Simplified Int8Variable quantization"; the readings
    are in the C file.  forward_outlier / backward_outlier compose them into
    the layer (the rebuilt kernel in the activation dtype, unquantized
    activations; numpy fp64 matmuls as the products).
  * quantize_weight_int4 / unpack_int4 / merge_int4 -- packed 4-bit kernels:
    keras-llm-light, "Simplified Int4Variable quantization" (two int4 values
    per int8 byte) and the 4-bit thread; the readings are in the C file.

  * float8 (submodule ``oracle.float8``, numpy) -- the float8 training
    recipe, "Introduce float8 training" (Keras PR 19488): E4M3 / E5M2
    codes, delayed scaling from an amax history, the float8 Dense layer's
    forward and backward; its readings are in the submodule's header.

Pins: every routine here is checked by ``tests/test_oracle_pins.py`` against
closed forms, brute force, finite differences and printed values (see
``tests/golden/``); the float8 submodule by ``tests/test_oracle_float8.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qlora_oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")
_LOCK = threading.Lock()
_LIB = None

_CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
           "-shared", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile the C oracle into ``liboracle.so`` (gcc).  Returns its path."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _lib():
    global _LIB
    with _LOCK:
        if _LIB is None:
            build()
            lib = ctypes.CDLL(_SO)
            P = ctypes.c_void_p
            L = ctypes.c_long
            D = ctypes.c_double
            F = ctypes.c_float
            lib.orc_set_threads.argtypes = [ctypes.c_int]
            lib.orc_get_threads.restype = ctypes.c_int
            lib.orc_quantize_weight.argtypes = [P, L, L, P, P]
            lib.orc_quantize_rows.argtypes = [P, L, L, P, P]
            lib.orc_int8_matmul.argtypes = [P, P, L, L, L, P]
            lib.orc_int8_matmul.restype = L
            lib.orc_lora_down.argtypes = [P, P, L, L, L, P]
            lib.orc_forward.argtypes = [L, L, L, D, P, P, P, P, P, P, P]
            lib.orc_backward.argtypes = [L, L, L, L, D, P, P, P, P, P, P,
                                         ctypes.c_int, P, P, P, P, P]
            lib.orc_merge.argtypes = [P, P, P, P, L, L, L, F, P, P]
            lib.orc_quantize_weight_int4.argtypes = [P, L, L, P, P]
            lib.orc_unpack_int4.argtypes = [P, L, L, P]
            lib.orc_merge_int4.argtypes = [P, P, P, P, L, L, L, F, P, P]
            lib.orc_percentile.argtypes = [P, L, D]
            lib.orc_percentile.restype = D
            lib.orc_round_fp16.argtypes = [D]
            lib.orc_round_fp16.restype = D
            lib.orc_quantize_outlier_int8.argtypes = [P, L, P, P, P, P]
            lib.orc_quantize_outlier_int8.restype = L
            lib.orc_dequantize_outlier_int8.argtypes = [P, P, P, L, F, F, P]
            lib.orc_round_bf16.argtypes = [D]
            lib.orc_round_bf16.restype = D
            lib.orc_round_bf16_array.argtypes = [P, L, P]
            _LIB = lib
    return _LIB


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def set_threads(n: int) -> None:
    _lib().orc_set_threads(int(n))


def get_threads() -> int:
    return int(_lib().orc_get_threads())


# --------------------------------------------------------------------------
# quantizers
# --------------------------------------------------------------------------
def quantize_weight(W):
    """W [K,N] float32 -> (Wq [N,K] int8, sw [N] float32), per output channel."""
    W = _c(W, np.float32)
    K, N = W.shape
    Wq = np.empty((N, K), np.int8)
    sw = np.empty((N,), np.float32)
    _lib().orc_quantize_weight(_p(W), K, N, _p(Wq), _p(sw))
    return Wq, sw


def quantize_rows(X):
    """X [M,K] float32 -> (Xq [M,K] int8, sx [M] float32), per row."""
    X = _c(X, np.float32)
    M, K = X.shape
    Xq = np.empty((M, K), np.int8)
    sx = np.empty((M,), np.float32)
    _lib().orc_quantize_rows(_p(X), M, K, _p(Xq), _p(sx))
    return Xq, sx


def int8_matmul(Xq, Wq):
    """acc[m,n] = sum_k Xq[m,k] Wq[n,k] in int64; raises if it leaves int32."""
    Xq = _c(Xq, np.int8)
    Wq = _c(Wq, np.int8)
    M, K = Xq.shape
    N, K2 = Wq.shape
    if K != K2:
        raise ValueError("inner sizes differ")
    acc = np.empty((M, N), np.int32)
    bad = _lib().orc_int8_matmul(_p(Xq), _p(Wq), M, N, K, _p(acc))
    if bad:
        raise OverflowError("%d accumulator entries leave the int32 range" % bad)
    return acc


# --------------------------------------------------------------------------
# layer
# --------------------------------------------------------------------------
def lora_down(X, A):
    X = _c(X, np.float64)
    A = _c(A, np.float64)
    M, K = X.shape
    r = A.shape[1]
    xA = np.empty((M, r), np.float64)
    _lib().orc_lora_down(_p(X), _p(A), M, K, r, _p(xA))
    return xA


def forward(X, Wq, sw, bias, A, B, alpha):
    """One int8-LoRA Dense forward.

    X holds exactly the values the layer sees (fp32, or bf16 widened).
    Returns a dict with the quantized input ``xq``/``sx``, the int32
    accumulator ``acc``, the LoRA down-projection ``xA`` and the fp64
    output ``y``.
    """
    X32 = _c(X, np.float32)
    M, K = X32.shape
    N = Wq.shape[0]
    r = A.shape[1]
    c = float(alpha) / float(r)
    Xq, sx = quantize_rows(X32)
    acc = int8_matmul(Xq, Wq)
    xA = lora_down(X32, A)
    Bd = _c(B, np.float64)
    bd = None if bias is None else _c(bias, np.float64)
    sw = _c(sw, np.float32)
    Y = np.empty((M, N), np.float64)
    _lib().orc_forward(M, N, r, c, _p(acc), _p(sx), _p(sw), _p(bd), _p(xA),
                       _p(Bd), _p(Y))
    return {"xq": Xq, "sx": sx, "acc": acc, "xA": xA, "y": Y}


def backward(X, dY, Wq, sw, A, B, alpha, want_dx=True, act="f32"):
    """One int8-LoRA Dense backward; returns dict G, dX, dA, dB, dbias (fp64).

    ``act`` is the activation dtype: the de-quantized kernel that enters dX is
    fl32(Wq * sw), rounded once more to bf16 when act == "bf16"."""
    Xd = _c(X, np.float64)
    dYd = _c(dY, np.float64)
    M, K = Xd.shape
    N = dYd.shape[1]
    r = A.shape[1]
    c = float(alpha) / float(r)
    Ad = _c(A, np.float64)
    Bd = _c(B, np.float64)
    Wq = _c(Wq, np.int8)
    sw = _c(sw, np.float32)
    G = np.empty((M, r), np.float64)
    dX = np.empty((M, K), np.float64) if want_dx else None
    dA = np.empty((K, r), np.float64)
    dB = np.empty((r, N), np.float64)
    db = np.empty((N,), np.float64)
    if act not in ("f32", "bf16"):
        raise ValueError(act)
    _lib().orc_backward(M, K, N, r, c, _p(Xd), _p(dYd), _p(Wq), _p(sw), _p(Ad),
                        _p(Bd), 1 if act == "bf16" else 0, _p(G), _p(dX), _p(dA), _p(dB),
                        _p(db))
    return {"G": G, "dX": dX, "dA": dA, "dB": dB, "dbias": db}


def merge(Wq, sw, A, B, alpha):
    """Lossy merge (fp32, fixed order) -> (Wq' [N,K] int8, sw' [N] float32)."""
    Wq = _c(Wq, np.int8)
    sw = _c(sw, np.float32)
    A = _c(A, np.float32)
    B = _c(B, np.float32)
    N, K = Wq.shape
    r = A.shape[1]
    c = np.float32(np.float32(alpha) / np.float32(r))
    Wq2 = np.empty_like(Wq)
    sw2 = np.empty_like(sw)
    _lib().orc_merge(_p(Wq), _p(sw), _p(A), _p(B), K, N, r, float(c), _p(Wq2), _p(sw2))
    return Wq2, sw2


# --------------------------------------------------------------------------
# packed int4 kernels (the int8 layer with 4-bit codes; readings in the C file)
# --------------------------------------------------------------------------
def quantize_weight_int4(W):
    """W [K,N] float32 (K even) -> (Wp [N, K/2] uint8 packed codes, sw [N] float32)."""
    W = _c(W, np.float32)
    K, N = W.shape
    if K % 2:
        raise ValueError("K must be even to pack two codes per byte")
    Wp = np.empty((N, K // 2), np.uint8)
    sw = np.empty((N,), np.float32)
    _lib().orc_quantize_weight_int4(_p(W), K, N, _p(Wp), _p(sw))
    return Wp, sw


def unpack_int4(Wp):
    """Wp [N, K/2] uint8 -> Wq [N, K] int8 codes (the layer's forward and
    backward are the int8 ones with these codes)."""
    Wp = _c(Wp, np.uint8)
    N, K2 = Wp.shape
    Wq = np.empty((N, 2 * K2), np.int8)
    _lib().orc_unpack_int4(_p(Wp), N, 2 * K2, _p(Wq))
    return Wq


def merge_int4(Wp, sw, A, B, alpha):
    """Lossy merge of an int4 layer -> (Wp' [N, K/2] uint8, sw' [N] float32)."""
    Wq = unpack_int4(Wp)
    sw = _c(sw, np.float32)
    A = _c(A, np.float32)
    B = _c(B, np.float32)
    N, K = Wq.shape
    r = A.shape[1]
    c = np.float32(np.float32(alpha) / np.float32(r))
    Wp2 = np.empty((N, K // 2), np.uint8)
    sw2 = np.empty_like(sw)
    _lib().orc_merge_int4(_p(Wq), _p(sw), _p(A), _p(B), K, N, r, float(c), _p(Wp2), _p(sw2))
    return Wp2, sw2


# --------------------------------------------------------------------------
# outlier-compensated int8 kernels (keras-llm-light; readings in the C file)
# --------------------------------------------------------------------------
def percentile(v, p):
    """Percentile p of the entries of v (linear interpolation), fp64."""
    v = _c(np.asarray(v).ravel(), np.float32)
    return float(_lib().orc_percentile(_p(v), v.size, float(p)))


def round_fp16(x):
    """Round an fp64 value to the nearest IEEE half, ties to even, as fp64."""
    return float(_lib().orc_round_fp16(float(x)))


def quantize_outlier_int8(W):
    """W (any shape) float32 -> dict of codes (uint8, W's shape), is_outlier
    (bool), outlier values (fp16 values as float32, 0 elsewhere), lo, hi,
    scale, bias and the outlier count."""
    W = _c(W, np.float32)
    n = W.size
    codes = np.empty(W.shape, np.uint8)
    is_out = np.empty(W.shape, np.uint8)
    vals = np.empty(W.shape, np.float32)
    par = np.empty(4, np.float32)
    count = _lib().orc_quantize_outlier_int8(_p(W), n, _p(codes), _p(is_out), _p(vals), _p(par))
    return {"codes": codes, "is_outlier": is_out.astype(bool), "values": vals, "lo": par[0],
            "hi": par[1], "scale": par[2], "bias": par[3], "count": int(count)}


def dequantize_outlier_int8(q):
    """The rebuilt fp32 kernel of a quantize_outlier_int8 result."""
    codes = _c(q["codes"], np.uint8)
    is_out = _c(q["is_outlier"].astype(np.uint8), np.uint8)
    vals = _c(q["values"], np.float32)
    W = np.empty(codes.shape, np.float32)
    _lib().orc_dequantize_outlier_int8(_p(codes), _p(is_out), _p(vals), codes.size,
                                       float(q["scale"]), float(q["bias"]), _p(W))
    return W


def outlier_kernel(q, act_dtype):
    """The kernel an outlier-compensated layer multiplies with: the rebuilt
    fp32 kernel of quantize_outlier_int8 (same shape as W, [K, N]), stored in
    the activation dtype (rounded to bf16 for bf16 layers), as fp64."""
    return to_act(dequantize_outlier_int8(q).astype(np.float64), act_dtype)


def forward_outlier(X, q, bias, A, B, alpha, act_dtype):
    """One outlier-compensated int8-LoRA Dense forward (keras-llm-light,
    "Simplified Int8Variable quantization": the kernel is rebuilt from its
    codes and outliers, and the activations are not quantized; "Parameter-
    efficient fine-tuning of GPT-2 with LoRA", "LoRA equation"):
    y = X . Wr + bias + c (X . A) . B in fp64, Wr = outlier_kernel(q, act).
    Returns dict xA, y."""
    Xd = np.asarray(X, np.float64)
    Wr = outlier_kernel(q, act_dtype)
    c = float(alpha) / float(A.shape[1])
    xA = lora_down(Xd, A)
    y = Xd @ Wr + c * (xA @ np.asarray(B, np.float64))
    if bias is not None:
        y = y + np.asarray(bias, np.float64)[None, :]
    return {"xA": xA, "y": y}


def backward_outlier(X, dY, q, A, B, alpha, act_dtype):
    """Its backward in fp64: G = dY B^T, dX = dY Wr^T + c G A^T,
    dA = c X^T G, dB = c (X A)^T dY, dbias = sum_m dY."""
    Xd = np.asarray(X, np.float64)
    dYd = np.asarray(dY, np.float64)
    Ad = np.asarray(A, np.float64)
    Bd = np.asarray(B, np.float64)
    c = float(alpha) / float(Ad.shape[1])
    Wr = outlier_kernel(q, act_dtype)
    G = dYd @ Bd.T
    return {"G": G, "dX": dYd @ Wr.T + c * (G @ Ad.T), "dA": c * (Xd.T @ G),
            "dB": c * (lora_down(Xd, A).T @ dYd), "dbias": dYd.sum(axis=0)}


def round_bf16(x):
    """Round fp64 values to the nearest bfloat16 (ties to even), as fp64."""
    x = _c(x, np.float64)
    y = np.empty_like(x)
    _lib().orc_round_bf16_array(_p(x), x.size, _p(y))
    return y


def to_act(y, act_dtype):
    """Store an fp64 result in the activation dtype ("f32" or "bf16"), as fp64."""
    if act_dtype == "bf16":
        return round_bf16(y)
    return np.asarray(y, np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# the MLP stack workload: Dense layers with a plain ReLU between them
# --------------------------------------------------------------------------
def mlp_stack(X, layers, dY, act_dtype):
    """Forward and backward through a stack of int8-LoRA Dense layers.

    ``layers`` is a list of dicts with Wq, sw, bias, A, B, alpha.  Every
    layer output is stored in ``act_dtype``; a ReLU follows every layer but
    the last.  ``dY`` is the gradient of the last layer's output.  Returns
    the final output, the gradient of the stack input, and per-layer dA/dB.
    """
    h = to_act(np.asarray(X, np.float64), act_dtype)
    inputs, pre = [], []
    n = len(layers)
    for i, L in enumerate(layers):
        inputs.append(h)
        out = forward(h, L["Wq"], L["sw"], L["bias"], L["A"], L["B"], L["alpha"])
        y = to_act(out["y"], act_dtype)
        pre.append(y)
        h = np.maximum(y, 0.0) if i < n - 1 else y
    y_final = h
    g = to_act(np.asarray(dY, np.float64), act_dtype)
    grads = [None] * n
    for i in range(n - 1, -1, -1):
        L = layers[i]
        if i < n - 1:
            g = np.where(pre[i] > 0.0, g, 0.0)
        b = backward(inputs[i], g, L["Wq"], L["sw"], L["A"], L["B"], L["alpha"],
                     want_dx=True, act=act_dtype)
        grads[i] = {"dA": b["dA"], "dB": b["dB"], "dbias": b["dbias"]}
        g = to_act(b["dX"], act_dtype)
    return {"y": y_final, "dX": g, "grads": grads, "inputs": inputs, "pre": pre}
