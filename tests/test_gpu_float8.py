"""GPU parity of the float8 recipe ("Introduce float8 training") against
oracle/float8.py: codes, scales and amax histories bit-exact, the float8
GEMMs and the layer's three products within tolerance.  Needs a B200."""
import numpy as np
import pytest
import torch

from oracle import float8 as f8

from parity import assert_close, to_np

pytestmark = pytest.mark.gpu

# fp32 sums of exact products of float8 values: norm-wise bound for fp32
# outputs (the sum's rounding, about sqrt(K) * 2^-24 of the largest partial
# sums, well inside this for K <= 8192)
F32_SUM_RTOL = 1e-4


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.fail("these tests need a CUDA device")
    from lora_fine_tuning_qlora_b200 import build
    build.build()
    from lora_fine_tuning_qlora_b200 import qlora
    return qlora


def _fmt(q, name):
    return q.FP8_E4M3 if name == f8.E4M3 else q.FP8_E5M2


@pytest.mark.parametrize("R,C,dtype,fmt,scale,L,with_qt", [
    # 8-aligned columns but rows % 16 != 0 with the transpose: the scalar kernel
    (300, 784, torch.bfloat16, f8.E4M3, 0.01, 7, True),
    (129, 1000, torch.float32, f8.E5M2, 1e-4, 1024, True),
    (1, 16, torch.float32, f8.E4M3, 1.0, 1, True),
    (37, 30, torch.bfloat16, f8.E4M3, 0.5, 3, True),   # columns not a multiple of 8
    # the 128 x 128 tiled kernel: whole and ragged tiles, both formats and types
    (64, 64, torch.bfloat16, f8.E5M2, 3.0, 1500, True),  # history longer than one block
    (304, 1000, torch.bfloat16, f8.E4M3, 0.01, 16, True),
    (2000, 520, torch.float32, f8.E5M2, 1e-3, 16, True),
    (1024, 384, torch.float32, f8.E4M3, 0.02, 16, True),
    (301, 136, torch.bfloat16, f8.E5M2, 2e-3, 4, False),  # no transpose: any row count
])
def test_quantize_state_bit_exact(q, R, C, dtype, fmt, scale, L, with_qt):
    rng = np.random.Generator(np.random.PCG64(R + C))
    T = (rng.standard_normal((R, C)) * rng.choice([1e-6, 1.0, 40.0, 1e4], (R, C))).astype(np.float32)
    Tt = torch.from_numpy(T).to(dtype).cuda()
    Tv = to_np(Tt).astype(np.float32)  # the values the kernel reads
    hist = (rng.random(L) * 5).astype(np.float32)
    hist[L // 2] = 0.0
    s_in = torch.tensor([scale], dtype=torch.float32, device="cuda")
    s_out = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    h = torch.from_numpy(hist).cuda()
    qq = torch.empty((R, C), dtype=torch.uint8, device="cuda")
    qt = torch.empty((C, R), dtype=torch.uint8, device="cuda") if with_qt else None
    q.qlora_fp8_quantize(Tt, _fmt(q, fmt), s_in, s_out, h, qq, qt)
    torch.cuda.synchronize()
    codes, amax, new = f8.step_tensor(Tv, {"scale": np.float32(scale), "history": hist}, fmt)
    np.testing.assert_array_equal(qq.cpu().numpy(), codes)
    if with_qt:
        np.testing.assert_array_equal(qt.cpu().numpy(), codes.T)
    assert to_np(s_out)[0] == new["scale"]
    np.testing.assert_array_equal(to_np(h), new["history"])


@pytest.mark.parametrize("R,C,dtype,fmt", [
    (4096, 520, torch.bfloat16, f8.E5M2),   # 32 row tiles; ragged last column strip
    (304, 1000, torch.float32, f8.E4M3),    # ragged row and column tiles
    (16, 8, torch.bfloat16, f8.E5M2),       # one partial tile
])
def test_quantize_colsum(q, R, C, dtype, fmt):
    """Codes, scale and history as without column sums; the sums within the
    fp32 bound R u sum_r |T[r, c]| (u = 2^-24, 2u allowed) of the exact
    column sums, and identical bits on a second call."""
    rng = np.random.Generator(np.random.PCG64(R * C))
    T = rng.normal(0, 1, (R, C)).astype(np.float32) + rng.normal(0, 3, C).astype(np.float32)[None, :]
    Tt = torch.from_numpy(T).to(dtype).cuda()
    Tv = to_np(Tt).astype(np.float64)
    hist = (rng.random(8) * 5).astype(np.float32)
    outs = []
    for _ in range(2):
        s_in = torch.tensor([0.05], device="cuda")
        s_out = torch.zeros(1, device="cuda")
        h = torch.from_numpy(hist).cuda()
        qq = torch.empty((R, C), dtype=torch.uint8, device="cuda")
        qt = torch.empty((C, R), dtype=torch.uint8, device="cuda")
        cs = torch.full((C,), np.nan, dtype=torch.float32, device="cuda")
        ws = torch.empty(q.qlora_fp8_colsum_workspace_bytes(R, C), dtype=torch.uint8, device="cuda")
        q.qlora_fp8_quantize_colsum(Tt, _fmt(q, fmt), s_in, s_out, h, qq, qt, cs, ws)
        torch.cuda.synchronize()
        outs.append((qq.cpu().numpy(), qt.cpu().numpy(), to_np(s_out)[0], to_np(h), to_np(cs)))
    codes, _, new = f8.step_tensor(Tv.astype(np.float32), {"scale": np.float32(0.05), "history": hist}, fmt)
    qq, qt, s1, h1, cs = outs[0]
    np.testing.assert_array_equal(qq, codes)
    np.testing.assert_array_equal(qt, codes.T)
    assert s1 == new["scale"]
    np.testing.assert_array_equal(h1, new["history"])
    ref = Tv.sum(axis=0)
    bound = R * 2.0 ** -23 * np.abs(Tv).sum(axis=0) + 1e-30
    assert np.all(np.abs(cs - ref) <= bound), np.abs(cs - ref).max()
    np.testing.assert_array_equal(outs[1][4], cs)


def test_zero_history_keeps_the_scale(q):
    T = torch.zeros((32, 32), dtype=torch.bfloat16, device="cuda")
    s_in = torch.tensor([0.5], device="cuda")
    s_out = torch.zeros(1, device="cuda")
    h = torch.zeros(16, device="cuda")
    qq = torch.empty((32, 32), dtype=torch.uint8, device="cuda")
    q.qlora_fp8_quantize(T, q.FP8_E4M3, s_in, s_out, h, qq)
    torch.cuda.synchronize()
    assert float(s_out[0]) == 0.5 and float(h.abs().max()) == 0.0 and int(qq.max()) == 0


@pytest.mark.parametrize("ws", [False, True])
@pytest.mark.parametrize("M,N,K,fa,fb,out", [
    (128, 128, 128, f8.E4M3, f8.E4M3, torch.bfloat16),
    (300, 520, 784, f8.E4M3, f8.E4M3, torch.bfloat16),   # ragged tiles and k-block
    (200, 264, 1024, f8.E5M2, f8.E4M3, torch.bfloat16),  # gradient x kernel
    (768, 384, 512, f8.E4M3, f8.E5M2, torch.float32),    # input^T x gradient
    (1, 16, 16, f8.E4M3, f8.E4M3, torch.float32),
    # CTA pairs (at least one 256 x 256 tile per two SMs): the last tile's
    # second half of rows and of columns wholly outside, ragged k-block
    (2148, 2100, 784, f8.E5M2, f8.E4M3, torch.bfloat16),
    # CTA pairs, several tiles per pair: both accumulator buffers and the
    # stage ring wrap
    (4096, 4096, 256, f8.E4M3, f8.E5M2, torch.float32),
])
def test_fp8_gemm(q, M, N, K, fa, fb, out, ws):
    """With ws, shapes that leave the CTA pairs a partial last wave (81 and
    256 tiles on 74 pairs) take the split of that wave: both halves'
    accumulators added by the second kernel."""
    rng = np.random.Generator(np.random.PCG64(M * N + K))
    A = rng.integers(0, 256, (M, K), dtype=np.uint8)
    B = rng.integers(0, 256, (N, K), dtype=np.uint8)
    # no NaN / infinity codes
    for X, fmt in ((A, fa), (B, fb)):
        bad = ~np.isfinite(f8.decode(X, fmt))
        X[bad] = 0x01
    sa, sb = np.float32(0.03125), np.float32(1.5)
    bias = rng.normal(0, 0.1, N).astype(np.float32)
    C = torch.full((M, N), float("nan"), dtype=out, device="cuda")
    args = (torch.from_numpy(A).cuda(), _fmt(q, fa), torch.from_numpy(B).cuda(), _fmt(q, fb),
            torch.tensor([sa], device="cuda"), torch.tensor([sb], device="cuda"),
            torch.from_numpy(bias).cuda(), C)
    if ws:
        need = q.qlora_fp8_gemm_workspace_bytes(M, N, K)
        w = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")
        q.qlora_fp8_gemm_ws(*args, w)
    else:
        q.qlora_fp8_gemm(*args)
    torch.cuda.synchronize()
    da, db = f8.decode(A, fa), f8.decode(B, fb)
    sab = np.float64(sa) * np.float64(sb)
    ref = (da @ db.T) * sab + bias[None, :]
    got = to_np(C)
    # per element: the fp32 sum of K exact products errs by at most
    # K u sum_k |a_k b_k| in any order (u = 2^-24; 2u allowed), then one
    # rounding to the output type (2^-8 relative for bf16, 2^-23 for fp32)
    sum_abs = (np.abs(da) @ np.abs(db).T) * sab
    out_u = 2.0 ** -8 if out == torch.bfloat16 else 2.0 ** -23
    tol = K * 2.0 ** -23 * sum_abs + out_u * np.abs(ref) + 1e-30
    bad = np.abs(got - ref) > tol
    assert not bad.any(), (int(bad.sum()), np.argwhere(bad)[0])


@pytest.mark.parametrize("M,N,K,out", [(300, 520, 784, torch.bfloat16), (2148, 2100, 784, torch.float32)])
def test_fp8_gemm_zero_operand_gives_the_bias(q, M, N, K, out):
    """A = 0: every output is its column's bias rounded once to the output
    type (0 * s + b is exact), so a bias taken from the wrong column, or an
    output written to the wrong place, shows bit for bit."""
    rng = np.random.Generator(np.random.PCG64(M + N))
    A = torch.zeros((M, K), dtype=torch.uint8, device="cuda")
    B = torch.from_numpy(rng.integers(0, 0x70, (N, K), dtype=np.uint8)).cuda()
    bias = torch.from_numpy(rng.normal(0, 1, N).astype(np.float32)).cuda()
    C = torch.full((M, N), 7.0, dtype=out, device="cuda")
    one = torch.ones(1, device="cuda")
    q.qlora_fp8_gemm(A, q.FP8_E4M3, B, q.FP8_E4M3, one, one, bias, C)
    torch.cuda.synchronize()
    want = bias.to(out)[None, :].expand(M, N)
    assert torch.equal(C, want)


@pytest.mark.parametrize("M,K,N,act", [(512, 768, 768, torch.bfloat16), (256, 1024, 320, torch.float32)])
def test_float8_dense_three_steps(q, M, K, N, act):
    """Three training steps of the float8 layer, each checked against the
    oracle carrying the same delayed-scaling state: codes of X, W, dY and
    the states bit-exact; Y, dX, dW, dbias within tolerance."""
    from lora_fine_tuning_qlora_b200.float8 import Float8Dense
    rng = np.random.Generator(np.random.PCG64(M + K + N))
    W = rng.normal(0, 0.05, (K, N)).astype(np.float32)
    bias = rng.normal(0, 0.01, N).astype(np.float32)
    L = 16
    lay = Float8Dense(torch.from_numpy(W).cuda(), torch.from_numpy(bias).cuda(), act, history_len=L)
    st = {k: {"scale": np.float32(1.0), "history": np.zeros(L, np.float32)} for k in ("x", "w", "g")}
    actname = "bf16" if act == torch.bfloat16 else "f32"
    for step in range(3):
        X = torch.from_numpy(rng.normal(0, 1 + step, (M, K)).astype(np.float32)).to(act).cuda()
        dY = torch.from_numpy(rng.normal(0, 1e-2, (M, N)).astype(np.float32)).to(act).cuda()
        Y, ctx = lay.forward(X)
        g = lay.backward(ctx, dY)
        torch.cuda.synchronize()
        Xv, dYv = to_np(X).astype(np.float32), to_np(dY).astype(np.float32)
        Wv = to_np(lay.W).astype(np.float32)
        sx, sw, sg = st["x"]["scale"], st["w"]["scale"], st["g"]["scale"]
        xq, _, st["x"] = f8.step_tensor(Xv, st["x"], f8.E4M3)
        wq, _, st["w"] = f8.step_tensor(Wv, st["w"], f8.E4M3)
        gq, _, st["g"] = f8.step_tensor(dYv, st["g"], f8.E5M2)
        np.testing.assert_array_equal(ctx["Xq"].cpu().numpy(), xq)
        np.testing.assert_array_equal(lay.Wq.cpu().numpy(), wq)
        np.testing.assert_array_equal(g["Gq"].cpu().numpy(), gq)
        for k, s in (("x", lay.sx), ("w", lay.sw), ("g", lay.sg)):
            assert to_np(s.scale)[0] == st[k]["scale"], (step, k)
            np.testing.assert_array_equal(to_np(s.history), st[k]["history"])
        f = f8.forward(Xv, Wv, bias, sx, sw)
        b = f8.backward(Xv, Wv, dYv, sx, sw, sg)
        assert_close(to_np(Y), f["y"], actname, "Y step %d" % step)
        assert_close(to_np(g["dX"]), b["dX"], actname, "dX step %d" % step)
        err = np.abs(to_np(g["dW"]) - b["dW"]).max() / np.abs(b["dW"]).max()
        assert err <= F32_SUM_RTOL, (step, err)
        assert_close(to_np(g["dbias"]), b["dbias"], actname, "dbias step %d" % step)
        # a plain update of the master weights between steps
        lay.W.sub_(0.1 * g["dW"])
