"""Pins of the float8 oracle (oracle/float8.py) against the formats'
definitions, torch's float8 casts, closed forms and exact-grid products.
CPU only."""
import numpy as np
import pytest
import torch

from oracle import float8 as f8


@pytest.mark.parametrize("fmt", [f8.E4M3, f8.E5M2])
def test_every_finite_code_round_trips(fmt):
    codes = np.arange(256, dtype=np.uint8)
    vals = f8.decode(codes, fmt)
    keep = np.isfinite(vals) & (codes != 0x80)  # -0 encodes as +0
    np.testing.assert_array_equal(f8.encode(vals[keep], fmt), codes[keep])


def test_format_landmarks():
    e, g = f8.E4M3, f8.E5M2
    cases = [(e, 448.0, 0x7E), (e, 2.0 ** -9, 0x01), (e, 2.0 ** -6, 0x08), (e, 1.0, 0x38),
             (e, -2.0, 0xC0), (e, 0.0, 0x00), (g, 57344.0, 0x7B), (g, 2.0 ** -16, 0x01),
             (g, 2.0 ** -14, 0x04), (g, 1.0, 0x3C), (g, -0.5, 0xB8)]
    for fmt, v, c in cases:
        assert int(f8.encode(np.array([v]), fmt)[0]) == c, (fmt, v)
        assert f8.decode(np.array([c], np.uint8), fmt)[0] == v, (fmt, c)
    assert np.isnan(f8.decode(np.array([0x7F], np.uint8), e)[0])
    assert np.isinf(f8.decode(np.array([0x7C], np.uint8), g)[0])


def test_ties_go_to_the_even_code():
    e, g = f8.E4M3, f8.E5M2
    # halfway between neighbours: the code with mantissa LSB 0 wins
    assert int(f8.encode(np.array([1.0625]), e)[0]) == 0x38     # 1.0 | 1.125
    assert int(f8.encode(np.array([1.1875]), e)[0]) == 0x3A     # 1.125 | 1.25
    assert int(f8.encode(np.array([3 * 2.0 ** -10]), e)[0]) == 0x02  # 2^-9 | 2^-8 (subnormals)
    assert int(f8.encode(np.array([1.125]), g)[0]) == 0x3C      # 1.0 | 1.25
    assert int(f8.encode(np.array([-1.375]), g)[0]) == 0xBE     # -1.25 | -1.5
    # just off the midpoint goes to the nearer value
    assert int(f8.encode(np.array([1.0625 + 1e-9]), e)[0]) == 0x39


@pytest.mark.parametrize("fmt,tdt", [(f8.E4M3, torch.float8_e4m3fn), (f8.E5M2, torch.float8_e5m2)])
def test_encode_matches_torch_casts_in_range(fmt, tdt):
    """torch's float8 casts (round to nearest even) agree on values inside
    the format's range, normal and subnormal."""
    rng = np.random.Generator(np.random.PCG64(8))
    x = np.concatenate([rng.normal(0, 1, 4000) * s for s in (1e-4, 1e-2, 1.0, 30.0, 300.0)])
    x = np.clip(x, -f8.MAX[fmt], f8.MAX[fmt]).astype(np.float32)
    want = torch.from_numpy(x).to(tdt).view(torch.uint8).numpy()
    got = f8.encode(x.astype(np.float64), fmt)
    # both of torch's zeros are acceptable for tiny negatives that round to zero
    diff = got != want
    assert np.all((want[diff] == 0x80) & (got[diff] == 0x00)), x[diff][:5]


def test_quantize_saturates_and_divides_once():
    q = f8.quantize(np.array([1000.0, -1e9, 3.0, 0.0], np.float32), 1.0, f8.E4M3)
    np.testing.assert_array_equal(q, [0x7E, 0xFE, 0x44, 0x00])
    # with scale 2 a grid value times 2 comes back exactly
    grid = f8.decode(np.arange(0x7F, dtype=np.uint8), f8.E4M3)
    t = (grid * 2.0).astype(np.float32)
    np.testing.assert_array_equal(f8.decode(f8.quantize(t, 2.0, f8.E4M3), f8.E4M3) * 2.0, t)
    # the division is fp32: 1/3 of 3.0 is fl32(1.0)
    assert f8.quantize(np.array([3.0], np.float32), np.float32(3.0), f8.E4M3)[0] == 0x38


def test_delayed_scaling_state():
    st = {"scale": np.float32(1.0), "history": np.array([0.0, 3.0, 1.0], np.float32)}
    q, amax, new = f8.step_tensor(np.array([[5.0, -2.0]], np.float32), st, f8.E4M3)
    assert amax == 5.0
    # the new scale comes from the history before this step's entry
    assert new["scale"] == np.float32(3.0 / 448.0)
    np.testing.assert_array_equal(new["history"], [5.0, 0.0, 3.0])
    np.testing.assert_array_equal(q, f8.encode(np.array([[5.0, -2.0]]), f8.E4M3))
    # an all-zero history keeps the old scale; so does a non-finite one
    z = {"scale": np.float32(0.25), "history": np.zeros(4, np.float32)}
    assert f8.next_scale(z["history"], z["scale"], f8.E5M2) == np.float32(0.25)
    assert f8.next_scale(np.array([np.inf], np.float32), 0.5, f8.E4M3) == np.float32(0.5)
    assert f8.next_scale(np.array([57344.0 * 4], np.float32), 1.0, f8.E5M2) == 4.0


def test_layer_products_on_exact_grids():
    """With every operand on its format's grid and unit scales, the layer is
    the plain float layer: Y = X W + b, dX = dY W^T, dW = X^T dY."""
    rng = np.random.Generator(np.random.PCG64(9))
    g4 = f8.decode(np.arange(0x7F, dtype=np.uint8), f8.E4M3)
    g5 = f8.decode(np.arange(0x7C, dtype=np.uint8), f8.E5M2)
    g4 = g4[np.abs(g4) < 8]
    g5 = g5[np.abs(g5) < 8]
    X = rng.choice(g4, (6, 5)) * rng.choice([-1, 1], (6, 5))
    W = rng.choice(g4, (5, 4)) * rng.choice([-1, 1], (5, 4))
    dY = rng.choice(g5, (6, 4)) * rng.choice([-1, 1], (6, 4))
    b = rng.normal(0, 1, 4)
    f = f8.forward(X, W, b, 1.0, 1.0)
    np.testing.assert_allclose(f["y"], X @ W + b, rtol=0, atol=1e-12)
    g = f8.backward(X, W, dY, 1.0, 1.0, 1.0)
    np.testing.assert_allclose(g["dX"], dY @ W.T, rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dW"], X.T @ dY, rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dbias"], dY.sum(axis=0), rtol=0, atol=1e-12)
    # scales multiply straight through: X*2, W*4 with scales 2, 4 give 8 X W
    f2 = f8.forward(X * 2, W * 4, None, 2.0, 4.0)
    np.testing.assert_allclose(f2["y"], 8 * (X @ W), rtol=0, atol=1e-12)
