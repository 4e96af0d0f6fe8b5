"""EinsumDense equations as the Dense layer on flattened axes: the equation
analysis (CPU), the flattening pinned against numpy's einsum through the
oracle (CPU), and the C-ABI path against the oracle (GPU)."""
import numpy as np
import pytest
import torch

import oracle
from lora_fine_tuning_qlora_b200 import einsum

from parity import assert_close, to_np


@pytest.mark.parametrize("eq,batch,kept,contracted,free,flat", [
    ("btd,dnh->btnh", "", "bt", "d", "nh", True),      # query / key / value projections
    ("btnh,nhd->btd", "", "bt", "nh", "d", True),      # attention output
    ("abc,cde->abde", "", "ab", "c", "de", True),
    ("ab,bc->ac", "", "a", "b", "c", True),            # Dense
    ("ab,bcd->acd", "", "a", "b", "cd", True),         # the float8 PR's EinsumDense example
    ("abc,bd->acd", "", "ac", "b", "d", False),        # contraction on an interior input axis
    ("btd,dnh->bnth", "", "bt", "d", "nh", False),     # output axes permuted
    ("btd,hdn->btnh", "", "bt", "d", "nh", False),     # contraction on an interior kernel axis
    # the float8 PR's speed test: kernel slices along a and b, a batched GEMM
    ("abcde,aebf->adbcf", "ab", "dc", "e", "f", False),
])
def test_plan_splits_axes(eq, batch, kept, contracted, free, flat):
    p = einsum.plan(eq)
    assert (p.batch, p.kept, p.contracted, p.free) == (batch, kept, contracted, free)
    assert p.flat == flat
    assert einsum.supported(eq)
    # the permutations reorder the operands into [batch, kept, contracted],
    # [batch, contracted, free] and back from [batch, kept, free]
    assert "".join(p.x[i] for i in p.x_perm) == batch + kept + contracted
    assert "".join(p.w[i] for i in p.w_perm) == batch + contracted + free
    assert "".join((batch + kept + free)[i] for i in p.out_perm) == p.out


@pytest.mark.parametrize("eq", ["ab,cd->abcd",      # no contraction
                                "ab,bb->ab",        # repeated axis
                                "abc,bd->ad",       # c summed over without the kernel
                                "ab,bcd->ac",       # d summed over without the input
                                "ab,bc->acz",       # z in neither operand
                                "ab->b"])           # not two operands
def test_plan_rejects_other_equations(eq):
    assert not einsum.supported(eq)
    with pytest.raises(ValueError):
        einsum.plan(eq)


def _grid(rng, shape, scale):
    """Values on the int8 grid of their abs-max, so quantization is exact."""
    v = rng.integers(-127, 128, shape).astype(np.float32)
    v.reshape(-1)[0] = 127.0
    return v * np.float32(scale)


def _inv(perm):
    inv = [0] * len(perm)
    for d, q in enumerate(perm):
        inv[q] = d
    return inv


def _canonical_operands(p, sizes, rng, r):
    """Canonical-order operands on exact int8 grids: Xc [nb, M, K] (every row's
    abs-max 127 * 0.5), Wc [nb, K, N] (every column's abs-max 127 * 2^-7),
    A [nb, K, r], B [nb, r, N], bias [N]."""
    ext = lambda s_: int(np.prod([sizes[c] for c in s_])) if s_ else 1
    nb, M, K, N = ext(p.batch), ext(p.kept), ext(p.contracted), ext(p.free)
    Xc = _grid(rng, (nb, M, K), 0.5)
    Xc[:, :, 0] = 63.5
    Wc = _grid(rng, (nb, K, N), 2.0 ** -7)
    Wc[:, 0, :] = 127.0 * 2.0 ** -7
    A = rng.normal(0, 0.1, (nb, K, r))
    B = rng.normal(0, 0.1, (nb, r, N))
    bias = rng.normal(0, 0.1, (N,))
    return nb, M, K, N, Xc, Wc, A, B, bias


@pytest.mark.parametrize("eq,sizes", [
    ("btd,dnh->btnh", dict(b=2, t=3, d=8, n=4, h=5)),
    ("btnh,nhd->btd", dict(b=3, t=2, n=4, h=5, d=6)),
    ("abc,bd->acd", dict(a=3, b=8, c=2, d=5)),
    ("btd,dnh->bnth", dict(b=2, t=3, d=8, n=4, h=5)),
    ("btd,hdn->btnh", dict(b=2, t=3, d=8, n=4, h=5)),
    ("abcde,aebf->adbcf", dict(a=2, b=3, c=2, d=3, e=8, f=4)),
])
def test_canonical_layout_matches_numpy_einsum(eq, sizes):
    """The batched Dense layer on the canonical operands (oracle, one call per
    batch slice), moved back to the equation's output order, equals numpy's
    einsum of the float layer.  Operands sit on exact int8 grids, so both
    quantizations are exact and only the axis bookkeeping is under test."""
    rng = np.random.Generator(np.random.PCG64(4))
    p = einsum.plan(eq)
    r = 2
    alpha = 4.0
    nb, M, K, N, Xc, Wc, A, B, bias = _canonical_operands(p, sizes, rng, r)
    shp = lambda s_: tuple(sizes[c] for c in s_)
    # the equation's operands: canonical order moved back by the inverse permutations
    X = Xc.reshape(shp(p.batch + p.kept + p.contracted)).transpose(_inv(p.x_perm))
    W = Wc.reshape(shp(p.batch + p.contracted + p.free)).transpose(_inv(p.w_perm))
    assert X.shape == shp(p.x) and W.shape == shp(p.w)
    Yc = np.empty((nb, M, N))
    for b in range(nb):
        Wq, sw = oracle.quantize_weight(np.ascontiguousarray(Wc[b]))
        Yc[b] = oracle.forward(np.ascontiguousarray(Xc[b]), Wq, sw, bias, A[b], B[b], alpha)["y"]
    Y = Yc.reshape(shp(p.batch + p.kept + p.free)).transpose(p.out_perm)
    # numpy: the float layer plus the per-slice low-rank term, slice by slice
    ref = np.einsum(eq, X.astype(np.float64), W.astype(np.float64))
    lora_c = np.einsum("bmk,bkr,brn->bmn", Xc.astype(np.float64), A, B) * (alpha / r)
    canon = shp(p.batch + p.kept + p.free)
    bias_c = np.broadcast_to(bias.reshape((1,) * len(p.batch + p.kept) + shp(p.free)), canon)
    ref = ref + (bias_c + lora_c.reshape(canon)).transpose(p.out_perm)
    np.testing.assert_allclose(Y, ref, rtol=1e-12, atol=1e-9)


@pytest.fixture(scope="module")
def built():
    from lora_fine_tuning_qlora_b200 import build
    build.build()


@pytest.mark.gpu
@pytest.mark.parametrize("shape,perm", [((3, 5, 7), (2, 0, 1)), ((2, 3, 4, 5, 6), (0, 3, 1, 2, 4)),
                                        ((64, 96), (1, 0)), ((1, 1, 9), (2, 1, 0))])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32, torch.int8])
def test_permute_kernel_bit_exact(built, shape, perm, dtype):
    if not torch.cuda.is_available():
        pytest.fail("this test needs a CUDA device")
    from lora_fine_tuning_qlora_b200 import qlora
    g = torch.Generator().manual_seed(3)
    src = (torch.randn(shape, generator=g) * 50).to(dtype).cuda()
    dst = qlora.qlora_permute(src, perm)
    torch.cuda.synchronize()
    assert torch.equal(dst.cpu(), src.cpu().permute(*perm).contiguous())


@pytest.mark.gpu
@pytest.mark.parametrize("eq,sizes,act", [
    ("btd,dnh->btnh", dict(b=4, t=96, d=256, n=4, h=64), "bf16"),       # no copy
    ("btnh,nhd->btd", dict(b=4, t=96, n=4, h=64, d=256), "bf16"),       # no copy
    ("btd,dnh->bnth", dict(b=4, t=96, d=256, n=4, h=64), "bf16"),       # permuted output
    ("bdt,dnh->btnh", dict(b=2, d=256, t=80, n=2, h=64), "bf16"),       # interior contraction
    ("btd,hdn->btnh", dict(b=3, t=40, d=512, h=32, n=4), "f32"),        # interior kernel axis
    ("abcde,aebf->adbcf", dict(a=2, b=3, c=8, d=16, e=64, f=32), "bf16"),  # the speed test's form
])
def test_einsum_dense_matches_oracle(built, eq, sizes, act):
    """EinsumDense forward and backward through the C ABI against the oracle's
    Dense layer on the canonical operands, slice by slice."""
    if not torch.cuda.is_available():
        pytest.fail("this test needs a CUDA device")
    rng = np.random.Generator(np.random.PCG64(5))
    p = einsum.plan(eq)
    r = 4
    alpha = 8.0
    tdt = torch.bfloat16 if act == "bf16" else torch.float32
    shp = lambda s_: tuple(sizes[c] for c in s_)
    ext = lambda s_: int(np.prod(shp(s_))) if s_ else 1
    nb, M, K, N = ext(p.batch), ext(p.kept), ext(p.contracted), ext(p.free)
    W = rng.normal(0, 0.05, shp(p.w)).astype(np.float32)
    A = rng.uniform(-0.05, 0.05, (nb, K, r)).astype(np.float32)
    B = rng.normal(0, 0.02, (nb, r, N)).astype(np.float32)
    bias = rng.normal(0, 0.01, shp(p.free)).astype(np.float32)
    lay = einsum.EinsumDense(eq, torch.from_numpy(W).cuda(), r, alpha, tdt,
                             bias=torch.from_numpy(bias).cuda(), A=torch.from_numpy(A).cuda(),
                             B=torch.from_numpy(B).cuda())
    X = torch.from_numpy(rng.normal(0, 1, shp(p.x)).astype(np.float32)).to(tdt).cuda()
    dY = torch.from_numpy(rng.normal(0, 1, shp(p.out)).astype(np.float32)).to(tdt).cuda()
    ws_ = lay.workspace(X)
    Y, xA = lay.forward(X, ws_)
    g = lay.backward(X, dY, xA, ws_)
    torch.cuda.synchronize()
    assert tuple(Y.shape) == shp(p.out) and tuple(g["dX"].shape) == shp(p.x)
    # the oracle on the canonical operands (numpy transposes of the values the layer saw)
    Xc = to_np(X).transpose(p.x_perm).reshape(nb, M, K)
    dYc = to_np(dY).transpose(_inv(p.out_perm)).reshape(nb, M, N)
    Wc = W.transpose(p.w_perm).reshape(nb, K, N)
    Yc = to_np(Y).transpose(_inv(p.out_perm)).reshape(nb, M, N)
    dXc = to_np(g["dX"]).transpose(p.x_perm).reshape(nb, M, K)
    dA = to_np(g["dA"]).reshape(nb, K, r)
    dB = to_np(g["dB"]).reshape(nb, r, N)
    dbias_ref = np.zeros(N)
    for b in range(nb):
        Wq, sw = oracle.quantize_weight(np.ascontiguousarray(Wc[b]))
        fwd = oracle.forward(Xc[b], Wq, sw, bias.reshape(N), A[b], B[b], alpha)
        bwd = oracle.backward(Xc[b], dYc[b], Wq, sw, A[b], B[b], alpha, act=act)
        assert_close(Yc[b], fwd["y"], act, "Y[%d]" % b)
        assert_close(dXc[b], bwd["dX"], act, "dX[%d]" % b)
        assert_close(dA[b], bwd["dA"], act, "dA[%d]" % b)
        assert_close(dB[b], bwd["dB"], act, "dB[%d]" % b)
        dbias_ref += bwd["dbias"]
    assert_close(to_np(g["dbias"]).reshape(N), dbias_ref, act, "dbias")
    if not p.batch and len(p.free) >= 2:  # per-head B view [heads, r, head_dim] over the same storage
        ph = lay.b_per_head()
        assert ph.data_ptr() == lay.layer.B.data_ptr()
        np.testing.assert_array_equal(to_np(ph), np.swapaxes(B[0].reshape((r,) + shp(p.free)), 0, 1))
