"""Pins for the CPU oracle: closed forms, brute force, finite differences and
hand-worked values, none of which re-types the oracle's own formulas.

Each test names what fixes the expected value: a printed or hand-derived
number (``tests/golden/``), a library routine that the special case reduces
to, an error bound of the quantizer, or central differences of a forward.
"""
import math
import os

import numpy as np
import pytest

import oracle
from lora_fine_tuning_qlora_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


# --------------------------------------------------------------------------
# quantizer
# --------------------------------------------------------------------------
def _load_ties():
    rows = []
    with open(os.path.join(GOLDEN, "quantize_ties.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            _, vals, q, s = [p.strip() for p in line.split("|")]
            rows.append((np.array(vals.split(), np.float32),
                         np.array(q.split(), np.int8), np.float32(s)))
    return rows


@pytest.mark.parametrize("case", range(4))
def test_quantize_golden_ties(case):
    """Round-half-to-even on exact products (hand-derived fixture)."""
    v, q_exp, s_exp = _load_ties()[case]
    # as one input row
    Xq, sx = oracle.quantize_rows(v[None, :])
    np.testing.assert_array_equal(Xq[0], q_exp)
    assert sx[0] == s_exp
    # as one kernel column (output channel)
    Wq, sw = oracle.quantize_weight(v[:, None])
    np.testing.assert_array_equal(Wq[0], q_exp)
    assert sw[0] == s_exp


@pytest.mark.parametrize("dist", ["normal", "student_t3", "outliers", "uniform01", "tiny"])
def test_quantize_error_bound(dist):
    """|w - q*s| <= s/2 (plus fp32 slack), |q| <= 127, amax maps to +-127."""
    rng = _rng(1)
    K, N = 257, 33
    if dist == "normal":
        W = rng.normal(0, 0.02, (K, N))
    elif dist == "student_t3":
        W = np.clip(rng.standard_t(3.0, (K, N)) * 0.02, -1, 1)
    elif dist == "outliers":
        W = rng.normal(0, 0.02, (K, N))
        W.reshape(-1)[rng.choice(K * N, 20, replace=False)] *= 20
    elif dist == "uniform01":
        W = rng.random((K, N))
    else:
        W = rng.normal(0, 1e-30, (K, N))
    W = W.astype(np.float32)
    Wq, sw = oracle.quantize_weight(W)
    assert Wq.shape == (N, K) and sw.shape == (N,)
    Wd = W.astype(np.float64)
    amax = np.abs(Wd).max(axis=0)
    # scale is amax/127 to fp32 rounding
    np.testing.assert_allclose(sw.astype(np.float64), amax / 127.0, rtol=2 ** -23, atol=0)
    deq = Wq.T.astype(np.float64) * sw.astype(np.float64)[None, :]
    err = np.abs(Wd - deq)
    bound = sw.astype(np.float64)[None, :] * (0.5 + 2 ** -14)
    assert np.all(err <= bound)
    assert np.abs(Wq.astype(np.int32)).max() <= 127
    # the element attaining amax maps to exactly +-127 with the sign of w
    arg = np.abs(Wd).argmax(axis=0)
    for n in range(N):
        assert Wq[n, arg[n]] == (127 if W[arg[n], n] > 0 else -127)
    # signs agree wherever q != 0
    nz = Wq.T != 0
    assert np.all(np.sign(Wq.T[nz]) == np.sign(W[nz]))


def test_quantize_matches_exact_rounding_away_from_ties():
    """Away from half-way points, q is the nearest integer to w*127/amax."""
    rng = _rng(2)
    X = rng.normal(0, 1, (64, 300)).astype(np.float32)
    Xq, sx = oracle.quantize_rows(X)
    t = X.astype(np.float64) * 127.0 / np.abs(X.astype(np.float64)).max(axis=1, keepdims=True)
    far = np.abs(np.abs(t - np.floor(t)) - 0.5) > 1e-4
    np.testing.assert_array_equal(Xq[far], np.rint(t[far]).astype(np.int8))


def test_quantize_zero_row_and_column():
    """amax = 0 gives q = 0 and s = 0 (no NaN)."""
    X = np.zeros((3, 16), np.float32)
    X[1, 3] = -2.0
    Xq, sx = oracle.quantize_rows(X)
    assert sx[0] == 0 and sx[2] == 0 and np.all(Xq[0] == 0) and np.all(Xq[2] == 0)
    assert Xq[1, 3] == -127
    W = np.zeros((16, 2), np.float32)
    Wq, sw = oracle.quantize_weight(W)
    assert np.all(Wq == 0) and np.all(sw == 0)


# --------------------------------------------------------------------------
# int8 matmul
# --------------------------------------------------------------------------
@pytest.mark.parametrize("shape", [(1, 1, 1), (3, 5, 7), (17, 33, 65), (64, 96, 784)])
def test_int8_matmul_vs_numpy(shape):
    """Triple loop in int64 equals numpy's int64 matmul (library routine)."""
    M, N, K = shape
    rng = _rng(3)
    Xq = rng.integers(-127, 128, (M, K), dtype=np.int8)
    Wq = rng.integers(-127, 128, (N, K), dtype=np.int8)
    acc = oracle.int8_matmul(Xq, Wq)
    ref = Xq.astype(np.int64) @ Wq.astype(np.int64).T
    np.testing.assert_array_equal(acc.astype(np.int64), ref)


def test_int8_matmul_range_check():
    """K * 127^2 leaves int32 for K = 140000: the oracle refuses to wrap."""
    K = 140000
    Xq = np.full((1, K), 127, np.int8)
    Wq = np.full((1, K), 127, np.int8)
    with pytest.raises(OverflowError):
        oracle.int8_matmul(Xq, Wq)
    # and 16384 * 127^2 fits
    K = 16384
    acc = oracle.int8_matmul(np.full((1, K), -127, np.int8), np.full((1, K), 127, np.int8))
    assert acc[0, 0] == -K * 127 * 127


# --------------------------------------------------------------------------
# hand-worked layer
# --------------------------------------------------------------------------
def _load_tiny():
    vals = {}
    with open(os.path.join(GOLDEN, "tiny_layer.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            vals[key] = np.array([float(x) for x in rest])
    return vals


def test_tiny_layer_golden():
    g = _load_tiny()
    X = g["X"].reshape(1, 2).astype(np.float32)
    W = g["W"].reshape(2, 2).astype(np.float32)
    A = g["A"].reshape(2, 1)
    B = g["B"].reshape(1, 2)
    alpha = g["alpha"][0]
    Wq, sw = oracle.quantize_weight(W)
    np.testing.assert_array_equal(Wq.reshape(-1), g["Wq"].astype(np.int8))
    out = oracle.forward(X, Wq, sw, g["bias"], A, B, alpha)
    np.testing.assert_array_equal(out["xq"].reshape(-1), g["Xq"].astype(np.int8))
    np.testing.assert_array_equal(out["acc"].reshape(-1), g["acc"].astype(np.int32))
    # fp32 scales are rounded: relative slack of a few fp32 ulps
    np.testing.assert_allclose(out["y"].reshape(-1), g["y"], rtol=1e-6)
    b = oracle.backward(X, g["dY"].reshape(1, 2), Wq, sw, A, B, alpha)
    np.testing.assert_allclose(b["G"].reshape(-1), g["G"], rtol=1e-12)
    np.testing.assert_allclose(b["dX"].reshape(-1), g["dX"], rtol=1e-6)
    np.testing.assert_allclose(b["dA"].reshape(-1), g["dA"], rtol=1e-12)
    np.testing.assert_allclose(b["dB"].reshape(-1), g["dB"], rtol=1e-12)
    np.testing.assert_allclose(b["dbias"], g["dbias"], rtol=1e-12)
    Wq2, sw2 = oracle.merge(Wq, sw, A.astype(np.float32), B.astype(np.float32), alpha)
    np.testing.assert_array_equal(Wq2.reshape(-1), g["Wq_merged"].astype(np.int8))
    np.testing.assert_allclose(sw2, g["sw_merged"], rtol=2e-7)


def test_lora_param_count_golden():
    """dA and dB together hold the notebook's 6,144 trainable parameters."""
    with open(os.path.join(GOLDEN, "lora_param_count.txt")) as f:
        K, N, r, frozen, trainable = [int(x) for x in
                                      [l for l in f if not l.startswith("#")][0].split()]
    rng = _rng(4)
    X = rng.normal(0, 1, (2, K)).astype(np.float32)
    W = rng.normal(0, 0.02, (K, N)).astype(np.float32)
    Wq, sw = oracle.quantize_weight(W)
    A = rng.uniform(-0.01, 0.01, (K, r))
    B = rng.normal(0, 0.01, (r, N))
    b = oracle.backward(X, rng.normal(0, 1, (2, N)), Wq, sw, A, B, 8.0, want_dx=False)
    assert Wq.size == frozen
    assert b["dA"].size + b["dB"].size == trainable


# --------------------------------------------------------------------------
# forward: exact-grid special case reduces to a float matmul
# --------------------------------------------------------------------------
@pytest.mark.parametrize("shape", [(5, 7, 3, 2), (33, 130, 70, 4), (16, 256, 10, 8)])
def test_forward_exact_grid_equals_float_layer(shape):
    """Inputs on the int8 grid (row/column abs-max 127 * 2^e) quantize exactly,
    so the layer is the plain float LoRA Dense: X W + b + c (X A) B."""
    M, K, N, r = shape
    rng = _rng(5)
    X = rng.integers(-127, 128, (M, K)).astype(np.float32)
    X[:, 0] = 127.0
    X *= np.float32(0.5)  # scale 0.5: amax 63.5, 127/amax = 2 exactly
    W = rng.integers(-127, 128, (K, N)).astype(np.float32)
    W[1, :] = -127.0
    W *= np.float32(2.0 ** -7)
    Wq, sw = oracle.quantize_weight(W)
    A = rng.normal(0, 0.1, (K, r))
    B = rng.normal(0, 0.1, (r, N))
    bias = rng.normal(0, 0.1, N)
    alpha = 2.0 * r
    out = oracle.forward(X, Wq, sw, bias, A, B, alpha)
    Xd, Wd = X.astype(np.float64), W.astype(np.float64)
    ref = Xd @ Wd + bias[None, :] + (alpha / r) * ((Xd @ A) @ B)
    np.testing.assert_allclose(out["y"], ref, rtol=1e-12, atol=1e-9)
    np.testing.assert_array_equal(out["xq"].astype(np.float64) * 0.5, Xd)


def test_forward_B_zero_is_base_layer():
    """B = 0 (the LoRA initialisation of B) gives exactly the base layer, dA = 0."""
    rng = _rng(6)
    M, K, N, r = 9, 40, 12, 4
    X = rng.normal(0, 1, (M, K)).astype(np.float32)
    W = rng.normal(0, 0.02, (K, N)).astype(np.float32)
    Wq, sw = oracle.quantize_weight(W)
    A = rng.uniform(-0.1, 0.1, (K, r))
    bias = rng.normal(0, 0.01, N)
    out = oracle.forward(X, Wq, sw, bias, A, np.zeros((r, N)), 32.0)
    base = oracle.forward(X, Wq, sw, bias, np.zeros((K, 1)), np.zeros((1, N)), 1.0)
    np.testing.assert_array_equal(out["y"], base["y"])
    dY = rng.normal(0, 1, (M, N))
    b0 = oracle.backward(X, dY, Wq, sw, A, np.zeros((r, N)), 32.0)
    assert np.all(b0["dA"] == 0.0) and np.all(b0["G"] == 0.0)
    bb = oracle.backward(X, dY, Wq, sw, np.zeros((K, 1)), np.zeros((1, N)), 1.0)
    np.testing.assert_array_equal(b0["dX"], bb["dX"])


def test_rank_one_adapter_is_an_outer_product_update():
    """r = 1: the adapter's contribution Y(B) - Y(B = 0) = c (X a) b is an
    outer product of two vectors, i.e. a matrix of rank exactly one (its
    second singular value vanishes), equal to numpy's outer product."""
    rng = _rng(7)
    M, K, N = 11, 24, 9
    X = rng.normal(0, 1, (M, K)).astype(np.float32)
    W = rng.normal(0, 0.05, (K, N)).astype(np.float32)
    Wq, sw = oracle.quantize_weight(W)
    a = rng.normal(0, 0.2, (K, 1))
    b = rng.normal(0, 0.2, (1, N))
    bias = rng.normal(0, 0.01, N)
    delta = (oracle.forward(X, Wq, sw, bias, a, b, 3.0)["y"]
             - oracle.forward(X, Wq, sw, bias, a, np.zeros((1, N)), 3.0)["y"])
    sv = np.linalg.svd(delta, compute_uv=False)
    assert sv[1] <= 1e-12 * sv[0]
    np.testing.assert_allclose(delta, 3.0 * np.outer(X.astype(np.float64) @ a[:, 0], b[0]),
                               rtol=1e-9, atol=1e-12)


def test_columns_at_plus_minus_amax_quantize_to_127():
    """A kernel whose every entry is +-a in its column quantizes to codes
    +-127 only, with scale a / 127."""
    rng = _rng(8)
    K, N = 33, 7
    amp = rng.uniform(0.1, 2.0, N).astype(np.float32)
    W = (np.where(rng.integers(0, 2, (K, N)) == 1, 1.0, -1.0) * amp[None, :]).astype(np.float32)
    Wq, sw = oracle.quantize_weight(W)
    np.testing.assert_array_equal(np.abs(Wq.astype(np.int32)), 127)
    np.testing.assert_array_equal(np.sign(Wq.T.astype(np.int32)), np.sign(W).astype(np.int32))
    np.testing.assert_allclose(sw.astype(np.float64), amp.astype(np.float64) / 127.0, rtol=2 ** -23)


def test_single_input_feature():
    """K = 1: each input row is its own abs-max, so it quantizes to +-127 (or
    0) and the base product is x * fl(q_w s_w) up to the fp32 roundings of the
    two scales; the adapter term is c x a b."""
    rng = _rng(9)
    M, N, r = 6, 5, 2
    X = rng.normal(0, 1, (M, 1)).astype(np.float32)
    X[2, 0] = 0.0
    W = rng.normal(0, 0.1, (1, N)).astype(np.float32)
    Wq, sw = oracle.quantize_weight(W)
    A = rng.normal(0, 0.3, (1, r))
    B = rng.normal(0, 0.3, (r, N))
    bias = rng.normal(0, 0.01, N)
    out = oracle.forward(X, Wq, sw, bias, A, B, 4.0)
    assert set(np.abs(out["xq"].astype(np.int32)).ravel().tolist()) <= {0, 127}
    assert out["xq"][2, 0] == 0 and out["sx"][2] == 0.0
    Xd = X.astype(np.float64)
    Wd = Wq.T.astype(np.float64) * sw.astype(np.float64)[None, :]
    ref = Xd @ Wd + bias[None, :] + (4.0 / r) * (Xd @ A) @ B
    np.testing.assert_allclose(out["y"], ref, rtol=1e-6, atol=1e-9)


# --------------------------------------------------------------------------
# backward: central differences
# --------------------------------------------------------------------------
def _loss(X, Wq, sw, bias, A, B, alpha, dY):
    return float(np.sum(oracle.forward(X, Wq, sw, bias, A, B, alpha)["y"] * dY))


@pytest.mark.parametrize("shape", [(3, 5, 4, 2), (4, 6, 3, 1)])
def test_backward_lora_grads_finite_differences(shape):
    """dA, dB, dbias against central differences of the actual forward."""
    M, K, N, r = shape
    rng = _rng(7)
    X = rng.normal(0, 1, (M, K)).astype(np.float32)
    W = rng.normal(0, 0.3, (K, N)).astype(np.float32)
    Wq, sw = oracle.quantize_weight(W)
    A = rng.normal(0, 0.5, (K, r))
    B = rng.normal(0, 0.5, (r, N))
    bias = rng.normal(0, 0.1, N)
    dY = rng.normal(0, 1, (M, N))
    alpha = 3.0
    g = oracle.backward(X, dY, Wq, sw, A, B, alpha)
    h = 1e-6
    for name, P, grad in (("A", A, g["dA"]), ("B", B, g["dB"]), ("bias", bias, g["dbias"])):
        fd = np.zeros_like(P)
        it = np.nditer(P, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            Pp, Pm = P.copy(), P.copy()
            Pp[idx] += h
            Pm[idx] -= h
            args = {"A": A, "B": B, "bias": bias}
            args[name] = Pp
            lp = _loss(X, Wq, sw, args["bias"], args["A"], args["B"], alpha, dY)
            args[name] = Pm
            lm = _loss(X, Wq, sw, args["bias"], args["A"], args["B"], alpha, dY)
            fd[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(grad, fd, rtol=1e-6, atol=1e-8, err_msg=name)


def test_backward_dx_finite_differences_of_straight_through_surrogate():
    """dX against central differences of X (Wq*sw)^T + b + c X A B, the
    forward with the input quantizer replaced by the identity."""
    M, K, N, r = 3, 5, 4, 2
    rng = _rng(8)
    X = rng.normal(0, 1, (M, K))
    W = rng.normal(0, 0.3, (K, N)).astype(np.float32)
    Wq, sw = oracle.quantize_weight(W)
    Wt = Wq.T.astype(np.float64) * sw.astype(np.float64)[None, :]
    A = rng.normal(0, 0.5, (K, r))
    B = rng.normal(0, 0.5, (r, N))
    bias = rng.normal(0, 0.1, N)
    dY = rng.normal(0, 1, (M, N))
    alpha = 6.0
    c = alpha / r

    def surrogate(Xv):
        return float(np.sum((Xv @ Wt + bias + c * (Xv @ A) @ B) * dY))

    g = oracle.backward(X, dY, Wq, sw, A, B, alpha)
    fd = np.zeros_like(X)
    h = 1e-6
    for m in range(M):
        for k in range(K):
            Xp, Xm = X.copy(), X.copy()
            Xp[m, k] += h
            Xm[m, k] -= h
            fd[m, k] = (surrogate(Xp) - surrogate(Xm)) / (2 * h)
    np.testing.assert_allclose(g["dX"], fd, rtol=1e-6, atol=1e-8)


def test_backward_dx_exact_grid_equals_float_layer_gradient():
    """On the exact grid the dequantized kernel is W itself: dX is the float
    layer's input gradient dY W^T + c dY B^T A^T (numpy matmuls)."""
    rng = _rng(9)
    M, K, N, r = 12, 48, 20, 4
    W = rng.integers(-127, 128, (K, N)).astype(np.float32)
    W[0, :] = 127.0
    W *= np.float32(2.0 ** -6)
    Wq, sw = oracle.quantize_weight(W)
    X = rng.normal(0, 1, (M, K))
    A = rng.normal(0, 0.2, (K, r))
    B = rng.normal(0, 0.2, (r, N))
    dY = rng.normal(0, 1, (M, N))
    g = oracle.backward(X, dY, Wq, sw, A, B, 8.0)
    ref = dY @ W.astype(np.float64).T + 2.0 * (dY @ B.T) @ A.T
    np.testing.assert_allclose(g["dX"], ref, rtol=1e-12, atol=1e-12)


def test_backward_dx_bf16_dequant_is_float_product_with_rounded_kernel():
    """For bf16 activations dX uses the de-quantized kernel rounded to bf16:
    it equals the float product dY Wb^T + c dY B^T A^T where Wb is fp32
    (q * s) rounded to bf16 by torch (library routine); on an exact grid
    the rounding is the identity and the two activation dtypes agree."""
    import torch
    rng = _rng(14)
    M, K, N, r = 7, 96, 40, 4
    W = rng.normal(0, 0.05, (K, N)).astype(np.float32)
    Wq, sw = oracle.quantize_weight(W)
    X = rng.normal(0, 1, (M, K))
    A = rng.normal(0, 0.2, (K, r))
    B = rng.normal(0, 0.2, (r, N))
    dY = rng.normal(0, 1, (M, N))
    g = oracle.backward(X, dY, Wq, sw, A, B, 8.0, act="bf16")
    w32 = Wq.T.astype(np.float32) * sw[None, :]
    wb = torch.from_numpy(np.ascontiguousarray(w32)).to(torch.bfloat16).double().numpy()
    ref = dY @ wb.T + 2.0 * (dY @ B.T) @ A.T
    np.testing.assert_allclose(g["dX"], ref, rtol=1e-12, atol=1e-12)
    # bf16 rounding really changed the kernel here (the pin is not vacuous)
    assert np.abs(wb - w32).max() > 0
    g32 = oracle.backward(X, dY, Wq, sw, A, B, 8.0, act="f32")
    assert np.abs(g32["dX"] - g["dX"]).max() > 0
    # exact grid: q * s is a short binary fraction, identical in both dtypes
    Wg = rng.integers(-127, 128, (K, N)).astype(np.float32)
    Wg[0, :] = 127.0
    Wg *= np.float32(2.0 ** -6)
    Wqg, swg = oracle.quantize_weight(Wg)
    gb = oracle.backward(X, dY, Wqg, swg, A, B, 8.0, act="bf16")
    gf = oracle.backward(X, dY, Wqg, swg, A, B, 8.0, act="f32")
    np.testing.assert_array_equal(gb["dX"], gf["dX"])


# --------------------------------------------------------------------------
# merge
# --------------------------------------------------------------------------
def test_merge_B_zero_roundtrips_codes():
    """With B = 0 the merge returns the same int8 codes; scales move <= 1 ulp."""
    rng = _rng(10)
    K, N, r = 300, 40, 4
    W = rng.standard_t(3.0, (K, N)).astype(np.float32) * np.float32(0.02)
    Wq, sw = oracle.quantize_weight(W)
    A = rng.uniform(-1, 1, (K, r)).astype(np.float32)
    Wq2, sw2 = oracle.merge(Wq, sw, A, np.zeros((r, N), np.float32), 8.0)
    np.testing.assert_array_equal(Wq2, Wq)
    np.testing.assert_allclose(sw2, sw, rtol=2 ** -23, atol=0)


def test_merge_within_requantization_bound_of_float_merge():
    """|q' s' - (q s + c A B)| <= s'/2 plus fp32 slack (lossy merge)."""
    rng = _rng(11)
    K, N, r = 257, 31, 4
    W = rng.normal(0, 0.02, (K, N)).astype(np.float32)
    Wq, sw = oracle.quantize_weight(W)
    A = rng.uniform(-1 / 16, 1 / 16, (K, r)).astype(np.float32)
    B = rng.normal(0, 0.05, (r, N)).astype(np.float32)
    alpha = 8.0
    Wq2, sw2 = oracle.merge(Wq, sw, A, B, alpha)
    exact = (Wq.T.astype(np.float64) * sw.astype(np.float64)[None, :]
             + (alpha / r) * (A.astype(np.float64) @ B.astype(np.float64)))
    deq = Wq2.T.astype(np.float64) * sw2.astype(np.float64)[None, :]
    amax = np.abs(exact).max(axis=0)
    bound = sw2.astype(np.float64)[None, :] * (0.5 + 2 ** -14) + amax[None, :] * 2 ** -20
    assert np.all(np.abs(deq - exact) <= bound)
    assert np.abs(Wq2.astype(np.int32)).max() == 127


def test_merged_vs_unmerged_output_bound():
    """The merged layer's output differs from the unmerged one by at most the
    kernel re-quantization error plus the LoRA branch's input-quantization
    error (Results footnote: merging into int8 is lossy)."""
    rng = _rng(12)
    M, K, N, r = 16, 200, 24, 4
    X = rng.normal(0, 1, (M, K)).astype(np.float32)
    W = rng.normal(0, 0.02, (K, N)).astype(np.float32)
    Wq, sw = oracle.quantize_weight(W)
    A = rng.uniform(-1 / 16, 1 / 16, (K, r)).astype(np.float32)
    B = rng.normal(0, 0.05, (r, N)).astype(np.float32)
    bias = rng.normal(0, 0.01, N)
    alpha = 8.0
    c = alpha / r
    un = oracle.forward(X, Wq, sw, bias, A, B, alpha)
    Wq2, sw2 = oracle.merge(Wq, sw, A, B, alpha)
    me = oracle.forward(X, Wq2, sw2, bias, np.zeros((K, 1)), np.zeros((1, N)), 1.0)
    xs = un["xq"].astype(np.float64) * un["sx"].astype(np.float64)[:, None]
    AB = A.astype(np.float64) @ B.astype(np.float64)
    amax_merged = np.abs(Wq.T * sw[None, :] + c * AB).max(axis=0)
    t1 = (np.abs(xs).sum(axis=1)[:, None]
          * (sw2.astype(np.float64)[None, :] * (0.5 + 2 ** -14) + amax_merged[None, :] * 2 ** -20))
    t2 = np.abs(c * (xs @ AB) - c * (un["xA"] @ B.astype(np.float64)))
    diff = np.abs(me["y"] - un["y"])
    assert np.all(diff <= t1 + t2 + 1e-12)
    # and the merge is really lossy here (not a vacuous bound)
    assert diff.max() > 0


# --------------------------------------------------------------------------
# bf16 storage and the MLP stack composition
# --------------------------------------------------------------------------
def test_round_bf16_matches_torch_for_fp32_values():
    """For fp32-representable values, direct fp64->bf16 RNE equals torch's
    fp32->bf16 conversion (library routine)."""
    import torch
    rng = _rng(13)
    x = np.concatenate([rng.normal(0, 1, 4000), rng.normal(0, 1e-30, 100),
                        rng.normal(0, 1e30, 100), [0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8]])
    x32 = x.astype(np.float32)
    ref = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.round_bf16(x32.astype(np.float64)), ref)
    # ties to even: 1 + 2^-8 -> 1, 1 + 3*2^-8 -> 1 + 2^-6
    assert oracle.round_bf16(np.array([1.0 + 2 ** -8]))[0] == 1.0
    assert oracle.round_bf16(np.array([1.0 + 3 * 2 ** -8]))[0] == 1.0 + 2 ** -6


def test_mlp_stack_single_layer_is_the_layer():
    spec = inputs.scaled(inputs.single_fp32(), M=8)
    d = inputs.layer_inputs(spec)
    Wq, sw = oracle.quantize_weight(d["W"])
    L = {"Wq": Wq, "sw": sw, "bias": d["bias"], "A": d["A"], "B": d["B"], "alpha": spec.alpha}
    st = oracle.mlp_stack(d["X"], [L], d["dY"], "f32")
    f = oracle.forward(d["X"], Wq, sw, d["bias"], d["A"], d["B"], spec.alpha)
    b = oracle.backward(d["X"], d["dY"], Wq, sw, d["A"], d["B"], spec.alpha)
    np.testing.assert_array_equal(st["y"], f["y"].astype(np.float32).astype(np.float64))
    np.testing.assert_array_equal(st["grads"][0]["dA"], b["dA"])
    np.testing.assert_array_equal(st["dX"], b["dX"].astype(np.float32).astype(np.float64))


def test_mlp_stack_relu_gates_the_gradient():
    """A unit whose pre-activation is negative passes no gradient back."""
    specs = inputs.mlp_stack(batch=4, hidden=32, depth=1, r=2, alpha=2.0, act="f32")
    d = inputs.mlp_stack_inputs(specs)
    layers = []
    for s, L in zip(specs, d["layers"]):
        Wq, sw = oracle.quantize_weight(L["W"])
        layers.append({"Wq": Wq, "sw": sw, "bias": L["bias"], "A": L["A"], "B": L["B"],
                       "alpha": s.alpha})
    st = oracle.mlp_stack(d["X"], layers, d["dY"], "f32")
    # gradient reaching layer 1's output = layer 2's dX masked by pre[1] > 0
    dz = st["pre"][1] > 0
    assert dz.any() and (~dz).any()
    # dB of layer 1 = c * xA^T (masked gradient): rows with a dead unit contribute 0
    # to that column; check via the column of a unit that is dead for every row
    dead_cols = np.where(~dz.any(axis=0))[0]
    for n in dead_cols:
        assert np.all(st["grads"][1]["dB"][:, n] == 0.0)


def test_input_generator_is_deterministic_and_shaped():
    s = inputs.dense4096(16)
    a = inputs.layer_inputs(inputs.scaled(s, K=256, N=128))
    b = inputs.layer_inputs(inputs.scaled(s, K=256, N=128))
    for k in a:
        if a[k] is not None:
            np.testing.assert_array_equal(a[k], b[k])
    assert a["X"].shape == (16, 256) and a["W"].shape == (256, 128)
    assert a["A"].shape == (256, 4) and a["B"].shape == (4, 128)
    assert np.abs(a["W"]).max() <= 1.0


# --------------------------------------------------------------------------
# packed int4 kernels
# --------------------------------------------------------------------------
def test_int4_byte_layout_by_hand():
    """One channel, K = 4: amax = 7/8 gives 7/amax = 8 exactly, so the codes
    are w * 8 = (-7, 3, 0, -1).  Packed two per byte, even k in the low
    nibble, as two's-complement nibbles: 0x39 (low 9 = -7, high 3) and 0xF0
    (low 0, high F = -1)."""
    W = np.array([[-7 / 8], [3 / 8], [0.0], [-1 / 8]], np.float32)
    Wp, sw = oracle.quantize_weight_int4(W)
    assert Wp.shape == (1, 2) and Wp.dtype == np.uint8
    assert Wp[0, 0] == 0x39 and Wp[0, 1] == 0xF0
    assert sw[0] == np.float32(0.125)
    np.testing.assert_array_equal(oracle.unpack_int4(Wp), [[-7, 3, 0, -1]])


def test_int4_ties_round_half_to_even():
    """amax = 7/8 (7/amax = 8): w = k/16 for odd k lands exactly on .5 and
    rounds to the even neighbour: 2.5 -> 2, 3.5 -> 4, -0.5 -> 0, 1.5 -> 2,
    -2.5 -> -2, 6.5 -> 6."""
    vals = [7 / 8, 2.5 / 8, 3.5 / 8, -0.5 / 8, 1.5 / 8, -2.5 / 8, 6.5 / 8, 0.0]
    W = np.array(vals, np.float32)[:, None]
    Wp, _ = oracle.quantize_weight_int4(W)
    np.testing.assert_array_equal(oracle.unpack_int4(Wp)[0], [7, 2, 4, 0, 2, -2, 6, 0])


def test_int4_every_code_survives_packing_in_both_nibbles():
    """Brute force over all 15 x 15 pairs of codes: a channel holding the
    pair (q0, q1) next to +-7 reference entries quantizes and unpacks to
    exactly those codes, in either position of the byte."""
    codes = list(range(-7, 8))
    cols = []
    for q0 in codes:
        for q1 in codes:
            cols.append([q0, q1, 7, -7])
    W = (np.array(cols, np.float32).T * np.float32(0.25))  # amax 7/4: 7/amax = 4 exactly
    Wp, sw = oracle.quantize_weight_int4(W)
    np.testing.assert_array_equal(oracle.unpack_int4(Wp), np.array(cols, np.int8))
    np.testing.assert_array_equal(sw, np.float32(0.25))


def test_int4_quantizer_properties():
    """Random channels: every nonzero channel reaches code +-7 at its abs-max,
    codes are monotone in w within a channel, every entry lies within half a
    step of its de-quantized value (plus the fp32 rounding of w * 7/amax),
    and an all-zero channel gets codes 0 and scale 0."""
    rng = _rng(11)
    K, N = 64, 12
    W = rng.standard_t(3, (K, N)).astype(np.float32) * 0.02
    W[:, 5] = 0.0
    Wp, sw = oracle.quantize_weight_int4(W)
    q = oracle.unpack_int4(Wp).astype(np.int32)  # [N, K]
    assert sw[5] == 0.0 and not q[5].any()
    for n in range(N):
        if n == 5:
            continue
        k = int(np.argmax(np.abs(W[:, n])))
        assert abs(q[n, k]) == 7 and np.sign(q[n, k]) == np.sign(W[k, n])
        order = np.argsort(W[:, n], kind="stable")
        assert (np.diff(q[n, order]) >= 0).all()
        amax = float(np.abs(W[:, n]).max())
        err = np.abs(W[:, n].astype(np.float64) - q[n] * float(sw[n]))
        assert (err <= (0.5 + 2 ** -20) * amax / 7).all()
    assert q.min() >= -7 and q.max() <= 7


def test_int4_merge_of_a_zero_adapter_keeps_the_codes():
    """B = 0: every merged entry is fl(q s), which re-quantizes to the same
    codes (the relative error of fl(q s) * fl(7 / fl(7 s)) is far below half
    a step), with a scale within one ulp of s."""
    rng = _rng(12)
    K, N, r = 32, 9, 4
    W = rng.normal(0, 0.05, (K, N)).astype(np.float32)
    Wp, sw = oracle.quantize_weight_int4(W)
    A = rng.normal(0, 0.3, (K, r)).astype(np.float32)
    Wp2, sw2 = oracle.merge_int4(Wp, sw, A, np.zeros((r, N), np.float32), 8.0)
    np.testing.assert_array_equal(oracle.unpack_int4(Wp2), oracle.unpack_int4(Wp))
    np.testing.assert_allclose(sw2, sw, rtol=2 ** -23)


def test_int4_merge_of_a_rank_one_power_of_two_adapter():
    """All codes 0 and a rank-one adapter of powers of two: the merged
    channel n is c a_k b_n (every product exact), so its codes are
    rne(7 a_k / max|a|) and its scale c |b_n| max|a| / 7."""
    K, N = 6, 3
    a = np.array([1.0, -0.5, 0.25, -1.0, 0.125, 0.5], np.float32)
    b = np.array([2.0, -0.25, 1.0], np.float32)
    Wp = np.zeros((N, K // 2), np.uint8)
    sw = np.full((N,), 0.01, np.float32)
    Wp2, sw2 = oracle.merge_int4(Wp, sw, a[:, None], b[None, :], 2.0)  # c = 2 / 1
    # 7 * a / max|a| = 7, -3.5, 1.75, -7, 0.875, 3.5 -> rne: 7, -4, 2, -7, 1, 4
    want = np.array([7, -4, 2, -7, 1, 4], np.int8)
    q = oracle.unpack_int4(Wp2)
    for n in range(N):
        np.testing.assert_array_equal(q[n], want * int(np.sign(b[n])))
        assert sw2[n] == np.float32(np.float32(2.0 * abs(b[n]) * 1.0) / np.float32(7.0))


# --------------------------------------------------------------------------
# outlier-compensated int8 kernels
# --------------------------------------------------------------------------
@pytest.mark.parametrize("p", [0.1, 99.9, 50.0, 0.0, 100.0, 37.25])
def test_percentile_is_numpys_linear_percentile(p):
    """The cutoffs use the order-statistic interpolation that numpy's
    percentile uses by default."""
    rng = _rng(21)
    for n in (1, 2, 999, 1001, 5000):
        v = rng.normal(0, 1, n).astype(np.float32)
        assert oracle.percentile(v, p) == pytest.approx(np.percentile(v.astype(np.float64), p),
                                                        rel=1e-12, abs=1e-12)


def test_round_fp16_is_ieee_half():
    """Round to nearest even into IEEE half: numpy's float16 conversion, on
    normal values, exact ties, subnormals and overflow."""
    rng = _rng(22)
    xs = list(rng.normal(0, 100, 2000)) + list(rng.normal(0, 1e-5, 500))
    xs += [1 + 2 ** -11, 1 + 3 * 2 ** -11, 2 ** -24 * 1.5, 2 ** -25, 65504.0, 65520.0, 1e6,
           -2 ** -14 * (1 + 2 ** -10), 0.0]
    with np.errstate(over="ignore"):  # 65520 and 1e6 overflow to inf, as they should
        for x in xs:
            assert oracle.round_fp16(x) == float(np.float16(x)), x


def _order_stat_outliers(n):
    """Entries strictly outside the 0.1th / 99.9th percentiles of n distinct
    values, per side: with h = (n - 1) / 1000, floor(h) + 1 when h is not an
    integer (the cutoff lies strictly between two order statistics), h when
    it is (the cutoff is an order statistic)."""
    h = (n - 1) / 1000
    return int(h) + 1 if h != int(h) else int(h)


@pytest.mark.parametrize("n", [500, 1001, 3200, 20001])
def test_outlier_count_and_exact_outliers(n):
    """The number of outliers matches the order-statistic count on both
    sides, the outliers come back as their fp16 values, and every other entry
    comes back within half a step (scale / 2) of itself, with codes in
    [0, 255]."""
    rng = _rng(23 + n)
    W = (rng.standard_t(3, n) * 0.05).astype(np.float32)
    q = oracle.quantize_outlier_int8(W)
    assert q["count"] == 2 * _order_stat_outliers(n)
    R = oracle.dequantize_outlier_int8(q)
    o = q["is_outlier"]
    assert (W[o] < q["lo"]).sum() == _order_stat_outliers(n)
    np.testing.assert_array_equal(R[o], np.array([float(np.float16(w)) for w in W[o]], np.float32))
    err = np.abs(R[~o].astype(np.float64) - W[~o])
    assert (err <= float(q["scale"]) * (0.5 + 2 ** -16) + 2 ** -22 * np.abs(W[~o])).all()
    assert q["codes"][o].max(initial=0) == 0
    assert q["codes"].max() <= 255


def test_outlier_cutoffs_that_are_entries_quantize_to_0_and_255():
    """n = 1001 values: (n - 1) / 1000 = 1, so the cutoffs are the second
    smallest and second largest entries; they quantize to 0 and 255, and the
    two extremes are the only outliers."""
    rng = _rng(24)
    W = rng.permutation(np.linspace(-1, 1, 1001)).astype(np.float32)
    W[np.argmin(W)] = -40.0
    W[np.argmax(W)] = 17.0
    q = oracle.quantize_outlier_int8(W)
    s = np.sort(W)
    assert q["lo"] == s[1] and q["hi"] == s[-2]
    assert q["count"] == 2 and set(W[q["is_outlier"]].tolist()) == {-40.0, 17.0}
    assert q["codes"][W == s[1]][0] == 0 and q["codes"][W == s[-2]][0] == 255


def test_constant_kernel_has_no_outliers_and_rebuilds_exactly():
    """All entries equal: both cutoffs are that value, the scale is 0, every
    code is 0 and the rebuilt kernel is the constant itself."""
    W = np.full((7, 9), -0.3125, np.float32)
    q = oracle.quantize_outlier_int8(W)
    assert q["count"] == 0 and q["scale"] == 0.0 and not q["codes"].any()
    np.testing.assert_array_equal(oracle.dequantize_outlier_int8(q), W)


# ---------------------------------------------------------------- outlier layer
def _outlier_layer(seed, K=24, N=20, M=7, r=3):
    rng = _rng(seed)
    W = (rng.normal(0, 0.02, size=(K, N))).astype(np.float32)
    W.reshape(-1)[rng.choice(K * N, size=3, replace=False)] *= 20.0
    X = rng.normal(size=(M, K))
    A = rng.uniform(-0.2, 0.2, size=(K, r)).astype(np.float32)
    B = rng.normal(0, 0.1, size=(r, N)).astype(np.float32)
    bias = rng.normal(0, 0.01, size=(N,)).astype(np.float32)
    dY = rng.normal(size=(M, N))
    return W, X, A, B, bias, dY


def test_outlier_layer_with_zero_adapter_is_the_rebuilt_kernel_product():
    """B = 0: the forward is X . Wr + bias, with Wr the rebuilt kernel (codes
    and fp16 outliers) checked entry by entry against the quantizer's own
    pieces: an outlier entry is its fp16 value, every other entry is
    bias + code * scale in fp32."""
    W, X, A, B, bias, _ = _outlier_layer(31)
    q = oracle.quantize_outlier_int8(W)
    f = oracle.forward_outlier(X, q, bias, A, np.zeros_like(B), 2.0, "f32")
    Wr = np.where(q["is_outlier"], q["values"],
                  np.float32(q["bias"]) + q["codes"].astype(np.float32) * np.float32(q["scale"]))
    np.testing.assert_allclose(f["y"], X @ Wr.astype(np.float64) + bias.astype(np.float64),
                               rtol=1e-12, atol=1e-12)
    # 480 entries: both cutoffs fall between the two most extreme order
    # statistics, so exactly one outlier on each side
    assert q["count"] == int(q["is_outlier"].sum()) == 2


def test_outlier_layer_gradients_are_central_differences():
    """The outlier layer is linear in X, A and B (nothing is quantized at run
    time), so dX, dA and dB equal central differences of the forward of the
    loss sum(dY * y) to rounding."""
    W, X, A, B, bias, dY = _outlier_layer(32, K=6, N=5, M=3, r=2)
    q = oracle.quantize_outlier_int8(W)
    alpha = 3.0
    g = oracle.backward_outlier(X, dY, q, A, B, alpha, "f32")
    A64, B64 = A.astype(np.float64), B.astype(np.float64)

    def loss(Xv, Av, Bv):
        Wr = oracle.outlier_kernel(q, "f32")
        y = Xv @ Wr + bias.astype(np.float64) + (alpha / A.shape[1]) * (Xv @ Av) @ Bv
        return float((dY * y).sum())

    h = 1e-6
    for name, base in (("dX", X.copy()), ("dA", A64.copy()), ("dB", B64.copy())):
        num = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            p, m = base.copy(), base.copy()
            p[idx] += h
            m[idx] -= h
            args_p = {"dX": (p, A64, B64), "dA": (X, p, B64), "dB": (X, A64, p)}[name]
            args_m = {"dX": (m, A64, B64), "dA": (X, m, B64), "dB": (X, A64, m)}[name]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(g[name], num, rtol=1e-6, atol=1e-8, err_msg=name)
    np.testing.assert_allclose(g["dbias"], dY.sum(axis=0), rtol=1e-12)


def test_outlier_kernel_in_bf16_is_the_rounded_rebuilt_kernel():
    """For bf16 layers the rebuilt kernel enters the products rounded to bf16
    (torch's conversion), like every operand of a bf16 layer."""
    import torch
    W, *_ = _outlier_layer(33)
    q = oracle.quantize_outlier_int8(W)
    Wr = oracle.dequantize_outlier_int8(q)
    ref = torch.from_numpy(Wr).to(torch.bfloat16).float().numpy().astype(np.float64)
    np.testing.assert_array_equal(oracle.outlier_kernel(q, "bf16"), ref)
