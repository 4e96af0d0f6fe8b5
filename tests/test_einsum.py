"""EinsumDense equations as the Dense layer on flattened axes: the equation
analysis (CPU), the flattening pinned against numpy's einsum through the
oracle (CPU), and the C-ABI path against the oracle (GPU)."""
import numpy as np
import pytest
import torch

import oracle
from lora_fine_tuning_qlora_b200 import einsum

from parity import assert_close, to_np


@pytest.mark.parametrize("eq,batch,contracted,free", [
    ("btd,dnh->btnh", "bt", "d", "nh"),     # query / key / value projections
    ("btnh,nhd->btd", "bt", "nh", "d"),     # attention output
    ("abc,cde->abde", "ab", "c", "de"),
    ("ab,bc->ac", "a", "b", "c"),           # Dense
    ("ab,bcd->acd", "a", "b", "cd"),        # the float8 PR's EinsumDense example
])
def test_plan_splits_axes(eq, batch, contracted, free):
    p = einsum.plan(eq)
    assert (p.batch, p.contracted, p.free) == (batch, contracted, free)
    assert einsum.supported(eq)


@pytest.mark.parametrize("eq", ["abc,bd->acd",      # contraction not on the trailing input axes
                                "btd,dnh->bnth",    # output axes permuted
                                "ab,cd->abcd",      # no contraction
                                "btd,hdn->btnh",    # contraction not on the leading kernel axes
                                "ab,bb->ab",        # repeated axis
                                # the float8 PR's speed test: the kernel shares axes a and b
                                # with the output, a batched GEMM with one kernel per (a, b)
                                "abcde,aebf->adbcf"])
def test_plan_rejects_other_equations(eq):
    assert not einsum.supported(eq)
    with pytest.raises(ValueError):
        einsum.plan(eq)


def _grid(rng, shape, scale):
    """Values on the int8 grid of their abs-max, so quantization is exact."""
    v = rng.integers(-127, 128, shape).astype(np.float32)
    v.reshape(-1)[0] = 127.0
    return v * np.float32(scale)


@pytest.mark.parametrize("eq,xs,ws", [("btd,dnh->btnh", (2, 3, 8), (8, 4, 5)),
                                      ("btnh,nhd->btd", (3, 2, 4, 5), (4, 5, 6)),
                                      ("abc,cde->abde", (2, 2, 6), (6, 3, 2))])
def test_flattening_matches_numpy_einsum(eq, xs, ws):
    """The Dense layer on the flattened operands (oracle) equals numpy's einsum
    of the float layer: X on its rows' int8 grid, W on its columns' grid (all
    of one column's entries share the column scale), so both quantizations are
    exact and only the axis bookkeeping is under test."""
    rng = np.random.Generator(np.random.PCG64(4))
    p = einsum.plan(eq)
    M, K, N, batch, contracted, free = einsum.flat_shapes(p, xs, ws)
    r = 2
    X = _grid(rng, xs, 0.5)
    Xf = X.reshape(M, K)
    Xf[:, 0] = 63.5  # every row's abs-max 127 * 0.5
    W = _grid(rng, ws, 2.0 ** -7)
    Wf = W.reshape(K, N)
    Wf[0, :] = 127.0 * 2.0 ** -7  # every column's abs-max 127 * 2^-7
    A = rng.normal(0, 0.1, contracted + (r,))
    B = rng.normal(0, 0.1, (r,) + free)
    bias = rng.normal(0, 0.1, free)
    alpha = 4.0
    Wq, sw = oracle.quantize_weight(Wf)
    y = oracle.forward(Xf, Wq, sw, bias.reshape(N), A.reshape(K, r), B.reshape(r, N), alpha)["y"]
    cx = p.contracted
    ref = (np.einsum(eq, X.astype(np.float64), W.astype(np.float64))
           + bias
           + (alpha / r) * np.einsum(p.batch + "z," + "z" + p.free + "->" + p.batch + p.free,
                                     np.einsum(p.batch + cx + "," + cx + "z->" + p.batch + "z",
                                               X.astype(np.float64), A), B))
    np.testing.assert_allclose(y.reshape(batch + free), ref, rtol=1e-12, atol=1e-9)


@pytest.fixture(scope="module")
def built():
    from lora_fine_tuning_qlora_b200 import build
    build.build()


@pytest.mark.gpu
@pytest.mark.parametrize("eq,xs,ws", [("btd,dnh->btnh", (4, 96, 256), (256, 4, 64)),
                                      ("btnh,nhd->btd", (4, 96, 4, 64), (4, 64, 256))])
def test_einsum_dense_matches_oracle(built, eq, xs, ws):
    """EinsumDense forward and backward through the C ABI against the oracle's
    Dense layer on the flattened operands, bf16 activations."""
    if not torch.cuda.is_available():
        pytest.fail("this test needs a CUDA device")
    rng = np.random.Generator(np.random.PCG64(5))
    p = einsum.plan(eq)
    M, K, N, batch, contracted, free = einsum.flat_shapes(p, xs, ws)
    r = 4
    W = rng.normal(0, 0.05, ws).astype(np.float32)
    A = rng.uniform(-0.05, 0.05, contracted + (r,)).astype(np.float32)
    B = rng.normal(0, 0.02, (r,) + free).astype(np.float32)
    bias = rng.normal(0, 0.01, free).astype(np.float32)
    lay = einsum.EinsumDense(eq, torch.from_numpy(W).cuda(), r, 8.0, torch.bfloat16,
                             bias=torch.from_numpy(bias).cuda(), A=torch.from_numpy(A).cuda(),
                             B=torch.from_numpy(B).cuda())
    X = torch.from_numpy(rng.normal(0, 1, xs).astype(np.float32)).to(torch.bfloat16).cuda()
    dY = torch.from_numpy(rng.normal(0, 1, batch + free).astype(np.float32)).to(torch.bfloat16).cuda()
    ws_ = lay.workspace(X)
    Y, xA = lay.forward(X, ws_)
    g = lay.backward(X, dY, xA, ws_)
    torch.cuda.synchronize()
    assert tuple(Y.shape) == batch + free and tuple(g["dX"].shape) == xs
    assert tuple(g["dA"].shape) == contracted + (r,) and tuple(g["dB"].shape) == (r,) + free
    Xo = to_np(X).reshape(M, K)   # the bf16 values the layer sees
    dYo = to_np(dY).reshape(M, N)
    Wq, sw = oracle.quantize_weight(W.reshape(K, N))
    fwd = oracle.forward(Xo, Wq, sw, bias.reshape(N), A.reshape(K, r), B.reshape(r, N), 8.0)
    bwd = oracle.backward(Xo, dYo, Wq, sw, A.reshape(K, r), B.reshape(r, N), 8.0, act="bf16")
    assert_close(to_np(Y).reshape(M, N), fwd["y"], "bf16", "Y")
    assert_close(to_np(g["dX"]).reshape(M, K), bwd["dX"], "bf16", "dX")
    assert_close(to_np(g["dA"]).reshape(K, r), bwd["dA"], "bf16", "dA")
    assert_close(to_np(g["dB"]).reshape(r, N), bwd["dB"], "bf16", "dB")
    if len(free) >= 2:  # per-head B view [heads, r, head_dim] over the same storage
        ph = lay.b_per_head()
        assert ph.data_ptr() == lay.layer.B.data_ptr()
        np.testing.assert_array_equal(to_np(ph), np.swapaxes(B, 0, 1))
