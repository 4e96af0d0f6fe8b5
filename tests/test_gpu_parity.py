"""GPU parity: the C-ABI path against the CPU oracle, element by element, on
seeded inputs shaped like the pages' workloads.  Needs a B200."""
import numpy as np
import pytest
import torch

import oracle
from lora_fine_tuning_qlora_b200 import inputs

from parity import assert_close, run_and_compare, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.fail("these tests need a CUDA device")
    from lora_fine_tuning_qlora_b200 import build
    build.build()
    from lora_fine_tuning_qlora_b200 import qlora
    oracle.set_threads(max(1, min(32, __import__("os").cpu_count() or 1)))
    return qlora


# ---------------------------------------------------------------- a0
@pytest.mark.parametrize("K,N", [(784, 128), (1024, 10), (768, 2304), (64, 48), (16, 1)])
def test_quantize_weight_bit_exact(q, K, N):
    rng = np.random.Generator(np.random.PCG64(K * 7 + N))
    W = rng.normal(0, 0.02, (K, N)).astype(np.float32)
    W[:, 0] = 0.0                      # an all-zero output channel
    if N > 1:
        W[3, 1] = 127.0 / 64           # exact .5 ties in that channel
        W[5, 1] = 2.5 / 64
        W[7, 1] = -3.5 / 64
    Wq, sw = q.quantize_weight(torch.from_numpy(W).cuda())
    Wq_o, sw_o = oracle.quantize_weight(W)
    np.testing.assert_array_equal(to_np(Wq), Wq_o)
    np.testing.assert_array_equal(to_np(sw).view(np.uint32), sw_o.view(np.uint32))


# ---------------------------------------------------------------- full layers
def test_single_fp32_layer(q):
    """The fp32 single-layer workload, every output compared."""
    run_and_compare(inputs.single_fp32(), q)


@pytest.mark.parametrize("M,K,N,r", [(300, 784, 520, 8), (129, 256, 136, 4), (1, 64, 16, 1),
                                     (200, 1040, 264, 16), (70, 128, 24, 64),
                                     (100, 4096, 136, 16), (1000, 1296, 264, 8),
                                     # few output tiles: split-K forward (clusters of 2..8 CTAs)
                                     (100, 2048, 520, 4), (16, 4096, 4096, 4), (250, 3072, 264, 8),
                                     (333, 1024, 1000, 8),
                                     # dX on CTA pairs (256 x 256 tiles): ragged M (the last
                                     # tile's second CTA wholly outside) and ragged K
                                     (850, 4736, 640, 4), (1100, 4736, 192, 16),
                                     # forward on CTA pairs: ragged M, N
                                     (1000, 1040, 4744, 8),
                                     # few tokens: tokens on the MMA's N, split-K clusters,
                                     # ragged channels and contraction
                                     (57, 1040, 200, 16), (64, 4096, 1000, 4), (9, 2048, 4096, 8)])
def test_bf16_layer_tiles_and_ragged_tails(q, M, K, N, r):
    spec = inputs.LayerSpec("ragged", M=M, K=K, N=N, r=r, alpha=2.0 * r, act="bf16",
                            x_dist="normal", w_dist="glorot", a_dist="he_uniform", b_std=0.01,
                            bias_dist="normal001", seed=M + K + N + r)
    run_and_compare(spec, q)


@pytest.mark.parametrize("M,K,N,r", [(96, 784, 128, 4), (33, 1040, 10, 8), (40, 12288, 72, 4)])
def test_fp32_layer_shapes(q, M, K, N, r):
    spec = inputs.LayerSpec("f32", M=M, K=K, N=N, r=r, alpha=r, act="f32", x_dist="normal",
                            w_dist="glorot", a_dist="he_uniform", b_std=0.01,
                            bias_dist="normal001", seed=M + N)
    run_and_compare(spec, q)


@pytest.mark.parametrize("i", [0, 1, 32])
def test_mlp_stack_layer_shapes(q, i):
    """784->1024, 1024->1024 and 1024->10 at batch 1024, every row."""
    run_and_compare(inputs.mlp_stack()[i], q)


@pytest.mark.parametrize("i", range(4))
def test_gpt2_base_projections(q, i):
    run_and_compare(inputs.gpt2_base()[i], q, sample_rows=192, seed=i)


@pytest.mark.parametrize("M", [512, 4096])
@pytest.mark.parametrize("i", range(7))
def test_gemma_2b_projections(q, M, i):
    spec = inputs.gemma_2b(M)[i]
    run_and_compare(spec, q, sample_rows=96, seed=i, check_merge=(M == 512))


@pytest.mark.parametrize("M", inputs.DENSE4096_M)
def test_dense4096_sweep(q, M):
    run_and_compare(inputs.dense4096(M), q, sample_rows=128, seed=M, check_merge=(M == 16))


# ---------------------------------------------------------------- edge cases
def _edge_spec(M, K, N, r, act="bf16", seed=5):
    return inputs.LayerSpec("edge", M=M, K=K, N=N, r=r, alpha=float(r), act=act, x_dist="normal",
                            w_dist="glorot", a_dist="he_uniform", b_std=0.01,
                            bias_dist="normal001", seed=seed)


def test_zero_rows_and_exact_ties(q):
    """All-zero input rows (scale 0), a row whose abs-max element is the only
    non-zero, and exact .5 ties in the input quantizer."""
    spec = _edge_spec(40, 256, 64, 4)
    d = inputs.layer_inputs(spec)
    X = d["X"]
    X[3, :] = 0.0
    X[7, :] = 0.0
    X[7, 11] = -1.5
    X[9, :] = 0.0
    X[9, 0] = 127.0 / 32.0                                     # 127/amax = 32 exactly
    X[9, 1:6] = np.array([2.5, 3.5, -0.5, 0.5, -1.5], np.float32) / 32.0
    from lora_fine_tuning_qlora_b200 import qlora
    layer_d = dict(d)
    layer_d["X"] = X
    W = torch.from_numpy(d["W"]).cuda()
    Wq, sw = q.quantize_weight(W)
    layer = q.Layer(Wq, sw, torch.from_numpy(d["bias"]).cuda(), torch.from_numpy(d["A"]).cuda(),
                    torch.from_numpy(d["B"]).cuda(), spec.alpha, torch.bfloat16)
    Xt = torch.from_numpy(X).to(torch.bfloat16).cuda()
    ws = q.workspace(layer.desc(), spec.M)
    Y, xA, (xq, sx, acc) = q.forward(layer, Xt, ws, debug=True)
    Wq_o, sw_o = oracle.quantize_weight(d["W"])
    f = oracle.forward(X, Wq_o, sw_o, d["bias"], d["A"], d["B"], spec.alpha)
    np.testing.assert_array_equal(to_np(xq), f["xq"])
    np.testing.assert_array_equal(to_np(sx).view(np.uint32), f["sx"].view(np.uint32))
    np.testing.assert_array_equal(to_np(acc), f["acc"])
    assert to_np(sx)[3] == 0 and np.all(to_np(xq)[3] == 0)
    np.testing.assert_array_equal(to_np(xq)[9, :6], [127, 2, 4, 0, 0, -2])
    assert to_np(xq)[7, 11] == -127
    assert_close(to_np(Y), f["y"], "bf16", "Y")


@pytest.mark.parametrize("M,K,r", [(16384, 4096, 4), (5000, 4096, 3), (8192, 3072, 4),
                                   (8200, 4096, 8), (4096, 768, 4), (12000, 2048, 2)])
def test_quantize_input_large_shapes(q, M, K, r):
    """a1 alone at the sizes where the staged input quantizer runs (rows
    streamed through shared memory by bulk copies), every row: codes and
    row scales bit-exact, xA within the bf16 tolerance.  Zero rows and a
    ragged last stage included."""
    rng = np.random.Generator(np.random.PCG64(M + K + r))
    X = inputs.round_to_act(rng.standard_normal((M, K), dtype=np.float32), "bf16")
    X[M // 2, :] = 0.0
    X[M - 1, :] = 0.0
    X[M - 1, K - 1] = 3.0
    A = rng.uniform(-1 / 64, 1 / 64, (K, r)).astype(np.float32)
    d = q.desc(K, 64, r, float(r), torch.bfloat16)
    Xt = torch.from_numpy(X).to(torch.bfloat16).cuda()
    At = torch.from_numpy(A).cuda()
    Xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty((M,), device="cuda")
    xA = torch.empty((M, r), device="cuda")
    q.qlora_quantize_input(d, M, Xt, At, Xq, sx, xA)
    torch.cuda.synchronize()
    assert q.qlora_device_status() == 0
    xq_o, sx_o = oracle.quantize_rows(X)
    np.testing.assert_array_equal(to_np(Xq), xq_o)
    np.testing.assert_array_equal(to_np(sx).view(np.uint32), sx_o.view(np.uint32))
    assert_close(to_np(xA), oracle.lora_down(X, A), "bf16", "xA")


def test_empty_batch(q):
    spec = _edge_spec(1, 64, 32, 4)
    d = inputs.layer_inputs(spec)
    from parity import device_layer
    layer = device_layer(spec, d, q)
    ws = q.workspace(layer.desc(), 1)
    X = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    Y = torch.empty((0, 32), dtype=torch.bfloat16, device="cuda")
    xA = torch.empty((0, 4), dtype=torch.float32, device="cuda")
    # M = 0: nothing to compute; forward is a no-op, backward gives zero gradients
    q.qlora_forward(layer.desc(), 0, torch.empty(16, dtype=torch.bfloat16, device="cuda"),
                    layer.Wq, layer.sw, layer.bias, layer.A, layer.B,
                    torch.empty(16, dtype=torch.bfloat16, device="cuda"),
                    torch.empty(4, device="cuda"), ws)
    dA = torch.full((64, 4), 7.0, device="cuda")
    dB = torch.full((4, 32), 7.0, device="cuda")
    db = torch.full((32,), 7.0, device="cuda")
    q.qlora_backward(layer.desc(), 0, torch.empty(16, dtype=torch.bfloat16, device="cuda"),
                     torch.empty(16, dtype=torch.bfloat16, device="cuda"), layer.Wq, layer.sw,
                     layer.A, layer.B, torch.empty(4, device="cuda"), None, dA, dB, db, ws)
    torch.cuda.synchronize()
    assert torch.all(dA == 0) and torch.all(dB == 0) and torch.all(db == 0)
    del X, Y, xA


def test_B_zero_gives_base_layer(q):
    """With the LoRA initialisation B = 0 the forward is the base layer and
    dA is exactly zero."""
    spec = inputs.scaled(_edge_spec(256, 512, 384, 4), b_std=0.0)
    out = run_and_compare(spec, q)
    assert torch.all(out["dA"] == 0)


def test_backward_is_deterministic(q):
    spec = inputs.gpt2_base(1024)[3]
    d = inputs.layer_inputs(spec)
    from parity import device_layer
    layer = device_layer(spec, d, q)
    X = torch.from_numpy(d["X"]).to(torch.bfloat16).cuda()
    dY = torch.from_numpy(d["dY"]).to(torch.bfloat16).cuda()
    ws = q.workspace(layer.desc(), spec.M)
    Y, xA = q.forward(layer, X, ws)
    r1 = q.backward(layer, X, dY, xA, ws)
    r2 = q.backward(layer, X, dY, xA, ws)
    for a, b in zip(r1, r2):
        assert torch.equal(a, b)


def test_device_status_is_clean(q):
    assert q.qlora_device_status() == 0


# ---------------------------------------------------------------- the MLP stack
@pytest.mark.slow
def test_mlp_stack_full(q):
    """The whole 33-layer MLP stack at batch 1024, forward and backward,
    against the oracle's stack (bf16 activations between layers)."""
    from lora_fine_tuning_qlora_b200 import stack
    specs = inputs.mlp_stack()
    data = inputs.mlp_stack_inputs(specs)
    net = stack.MLPStack.from_inputs(specs, data)
    out = net.step(torch.from_numpy(data["X"]).to(torch.bfloat16).cuda(),
                   torch.from_numpy(data["dY"]).to(torch.bfloat16).cuda())
    torch.cuda.synchronize()
    layers = []
    for s, L in zip(specs, data["layers"]):
        Wq, sw = oracle.quantize_weight(L["W"])
        layers.append({"Wq": Wq, "sw": sw, "bias": L["bias"], "A": L["A"], "B": L["B"], "alpha": s.alpha})
    ref = oracle.mlp_stack(data["X"], layers, data["dY"], "bf16")
    # Elementwise bound only: through 33 re-quantized layers a last-bit
    # difference of an intermediate bf16 activation moves an input code and
    # grows from layer to layer, so the composition is not held to the
    # norm-wise bound of a single layer (every single layer is, above).
    assert_close(to_np(out["y"]), ref["y"], "bf16", "stack Y", norm=False)
    assert_close(to_np(out["dX"]), ref["dX"], "bf16", "stack dX", norm=False)
    for i in range(len(specs)):
        assert_close(to_np(out["dA"][i]), ref["grads"][i]["dA"], "bf16", "dA[%d]" % i, norm=False)
        assert_close(to_np(out["dB"][i]), ref["grads"][i]["dB"], "bf16", "dB[%d]" % i, norm=False)


def test_step_level_calls_match_composite(q):
    """a1..a5 called one by one (G left in the workspace by a3, also
    materialised on request) give the composite forward/backward results."""
    spec = _edge_spec(200, 384, 264, 8, seed=11)
    d = inputs.layer_inputs(spec)
    from parity import device_layer
    layer = device_layer(spec, d, q)
    X = torch.from_numpy(d["X"]).to(torch.bfloat16).cuda()
    dY = torch.from_numpy(d["dY"]).to(torch.bfloat16).cuda()
    ws = q.workspace(layer.desc(), spec.M)
    Y, xA = q.forward(layer, X, ws)
    dX, dA, dB, db = q.backward(layer, X, dY, xA, ws)
    D = layer.desc()
    M = spec.M
    Xq = torch.empty((M, spec.K), dtype=torch.int8, device="cuda")
    sx = torch.empty((M,), device="cuda")
    xA2 = torch.empty_like(xA)
    Y2 = torch.empty_like(Y)
    q.qlora_quantize_input(D, M, X, layer.A, Xq, sx, xA2)
    q.qlora_gemm_forward(D, M, Xq, sx, layer.Wq, layer.sw, layer.bias, xA2, layer.B, Y2)
    dB2 = torch.empty_like(dB)
    db2 = torch.empty_like(db)
    G = torch.empty((M, spec.r), device="cuda")
    q.qlora_lora_grad_dy(D, M, dY, layer.B, xA2, dB2, db2, ws, G)
    dX2 = torch.empty_like(dX)
    q.qlora_gemm_dx(D, M, dY, layer.Wq, layer.sw, layer.A, dX2, ws)
    dA2 = torch.empty_like(dA)
    q.qlora_lora_grad_x(D, M, X, dA2, ws)
    torch.cuda.synchronize()
    for a, b in ((Y, Y2), (dX, dX2), (dA, dA2), (dB, dB2), (db, db2)):
        assert torch.equal(a, b)
    G_ref = oracle.backward(d["X"], d["dY"], *oracle.quantize_weight(d["W"]), d["A"], d["B"],
                            spec.alpha, want_dx=False)["G"]
    assert_close(to_np(G), G_ref, "bf16", "G")


@pytest.mark.parametrize("M,K,N,r,act", [(200, 384, 264, 8, "bf16"), (333, 784, 1024, 4, "bf16"),
                                          (96, 256, 10, 8, "bf16"), (64, 784, 128, 4, "f32"),
                                          (70, 128, 2304, 16, "bf16")])
def test_split_dy_pass_matches_grad_dy(q, M, K, N, r, act):
    """qlora_lora_g followed by qlora_lora_grad_b (on another stream) gives
    the results of qlora_lora_grad_dy: the same dB and dbias, and a
    workspace from which a4 and a5 give the same dX and dA; dB, dA and G
    also against the oracle."""
    spec = _edge_spec(M, K, N, r, act=act, seed=M + N)
    d = inputs.layer_inputs(spec)
    from parity import device_layer, act_torch
    layer = device_layer(spec, d, q)
    tdt = act_torch(act)
    X = torch.from_numpy(d["X"]).to(tdt).cuda()
    dY = torch.from_numpy(d["dY"]).to(tdt).cuda()
    D = layer.desc()
    ws1 = q.workspace(D, M)
    ws2 = q.workspace(D, M)
    _, xA = q.forward(layer, X, ws1)
    dB1 = torch.empty((r, N), device="cuda"); db1 = torch.empty((N,), device="cuda")
    q.qlora_lora_grad_dy(D, M, dY, layer.B, xA, dB1, db1, ws1)
    dB2 = torch.full((r, N), float("nan"), device="cuda")
    db2 = torch.full((N,), float("nan"), device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    q.qlora_lora_g(D, M, dY, layer.B, ws2)
    with torch.cuda.stream(side):
        q.qlora_lora_grad_b(D, M, dY, xA, dB2, db2, side)
    torch.cuda.current_stream().wait_stream(side)
    outs = []
    for ws in (ws1, ws2):
        dX = torch.empty((M, K), dtype=tdt, device="cuda")
        dA = torch.empty((K, r), device="cuda")
        q.qlora_gemm_dx(D, M, dY, layer.Wq, layer.sw, layer.A, dX, ws)
        q.qlora_lora_grad_x(D, M, X, dA, ws)
        outs.append((dX, dA))
    torch.cuda.synchronize()
    assert q.qlora_device_status() == 0
    assert torch.equal(dB1, dB2) and torch.equal(db1, db2)
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    ref = oracle.backward(oracle.to_act(d["X"], act), oracle.to_act(d["dY"], act),
                          *oracle.quantize_weight(d["W"]), d["A"], d["B"], spec.alpha,
                          want_dx=False, act=act)
    assert_close(to_np(dB2), ref["dB"], act, "dB")
    assert_close(to_np(db2), ref["dbias"], act, "dbias")
    assert_close(to_np(outs[1][1]), ref["dA"], act, "dA")


@pytest.mark.parametrize("M,K,N,r", [(1024, 1024, 1024, 8), (1000, 784, 264, 4), (3000, 256, 512, 16)])
def test_rank_pass_rows_setting(q, M, K, N, r):
    """With 256 and 1024 rows per CTA (and back at the default) the dB/dbias
    and dA passes still match the oracle, and two calls with the same
    setting agree bit for bit."""
    spec = _edge_spec(M, K, N, r, seed=M + 11 * N)
    d = inputs.layer_inputs(spec)
    from parity import device_layer
    layer = device_layer(spec, d, q)
    X = torch.from_numpy(d["X"]).to(torch.bfloat16).cuda()
    dY = torch.from_numpy(d["dY"]).to(torch.bfloat16).cuda()
    D = layer.desc()
    ws = q.workspace(D, M)
    _, xA = q.forward(layer, X, ws)
    q.qlora_lora_g(D, M, dY, layer.B, ws)
    ref = oracle.backward(oracle.to_act(d["X"], "bf16"), oracle.to_act(d["dY"], "bf16"),
                          *oracle.quantize_weight(d["W"]), d["A"], d["B"], spec.alpha,
                          want_dx=False, act="bf16")
    try:
        for rows in (256, 1024, 0):
            assert q.qlora_set_rank_pass_rows(rows) in (0, 256, 1024)
            outs = []
            for _ in range(2):
                dB = torch.full((r, N), float("nan"), device="cuda")
                db = torch.full((N,), float("nan"), device="cuda")
                dA = torch.full((K, r), float("nan"), device="cuda")
                q.qlora_lora_grad_b(D, M, dY, xA, dB, db)
                q.qlora_lora_grad_x(D, M, X, dA, ws)
                outs.append((dB, db, dA))
            torch.cuda.synchronize()
            assert q.qlora_device_status() == 0
            for a_, b_ in zip(*outs):
                assert torch.equal(a_, b_)
            dB, db, dA = outs[0]
            assert_close(to_np(dB), ref["dB"], "bf16", "dB rows=%d" % rows)
            assert_close(to_np(db), ref["dbias"], "bf16", "dbias rows=%d" % rows)
            assert_close(to_np(dA), ref["dA"], "bf16", "dA rows=%d" % rows)
    finally:
        q.qlora_set_rank_pass_rows(0)


@pytest.mark.parametrize("M,K,N,r,act", [(200, 384, 264, 8, "bf16"), (96, 256, 10, 8, "bf16"),
                                          (64, 784, 128, 4, "f32"), (300, 2048, 264, 8, "bf16"),
                                          (600, 8192, 256, 8, "bf16"), (2048, 512, 9216, 4, "bf16"),
                                          (48, 1024, 768, 8, "bf16")])
def test_fused_relu_entry_points(q, M, K, N, r, act):
    """qlora_gemm_forward_relu == qlora_relu(qlora_gemm_forward) and
    qlora_gemm_dx_relu == qlora_relu_backward(qlora_gemm_dx, X), bit for bit,
    on the tensor-core and CUDA-core paths."""
    spec = _edge_spec(M, K, N, r, act=act, seed=3 * M + N)
    d = inputs.layer_inputs(spec)
    from parity import device_layer, act_torch
    layer = device_layer(spec, d, q)
    tdt = act_torch(act)
    X = torch.from_numpy(d["X"]).to(tdt).cuda()
    X = torch.where(torch.arange(K, device="cuda") % 3 == 0, -X.abs(), X)  # plenty of X <= 0
    dY = torch.from_numpy(d["dY"]).to(tdt).cuda()
    D = layer.desc()
    ws = q.workspace(D, M)
    Xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty((M,), device="cuda")
    xA = torch.empty((M, r), device="cuda")
    q.qlora_quantize_input(D, M, X, layer.A, Xq, sx, xA)
    Y1 = torch.empty((M, N), dtype=tdt, device="cuda")
    Y2 = torch.empty_like(Y1)
    q.qlora_gemm_forward(D, M, Xq, sx, layer.Wq, layer.sw, layer.bias, xA, layer.B, Y1)
    q.qlora_relu(Y1)
    q.qlora_gemm_forward_relu(D, M, Xq, sx, layer.Wq, layer.sw, layer.bias, xA, layer.B, Y2)
    dB = torch.empty((r, N), device="cuda")
    q.qlora_lora_grad_dy(D, M, dY, layer.B, xA, dB, None, ws)
    dX1 = torch.empty((M, K), dtype=tdt, device="cuda")
    dX2 = torch.full_like(dX1, float("nan"))
    q.qlora_gemm_dx(D, M, dY, layer.Wq, layer.sw, layer.A, dX1, ws)
    q.qlora_relu_backward(dX1, X)
    q.qlora_gemm_dx_relu(D, M, dY, layer.Wq, layer.sw, layer.A, X, dX2, ws)
    torch.cuda.synchronize()
    assert q.qlora_device_status() == 0
    assert torch.equal(Y1, Y2)
    assert torch.equal(dX1, dX2)
    assert (Y2 >= 0).all() and (dX2[X <= 0] == 0).all()


def test_relu_kernels(q):
    """The stack's elementwise ReLU and its backward, aligned and unaligned."""
    rng = np.random.Generator(np.random.PCG64(21))
    for dtype in (torch.bfloat16, torch.float32):
        x = torch.from_numpy(rng.normal(0, 1, 1003).astype(np.float32)).to(dtype).cuda()
        for off in (0, 1):
            y = x[off:].clone() if off == 0 else x.clone()[off:]
            ref = torch.clamp(y.float(), min=0)
            q.qlora_relu(y)
            g = torch.ones_like(y)
            q.qlora_relu_backward(g, y)
            torch.cuda.synchronize()
            assert torch.equal(y.float(), ref)
            assert torch.equal(g.float(), (ref > 0).float())


# ---------------------------------------------------------------- packed int4
@pytest.mark.parametrize("K,N", [(1024, 1024), (768, 2304), (32, 10), (4096, 136)])
def test_int4_quantize_and_unpack_bit_exact(q, K, N):
    """The int4 quantizer and the unpack kernel against the oracle, byte for
    byte, on heavy-tailed kernels with a zero channel and exact .5 ties."""
    rng = np.random.Generator(np.random.PCG64(K + 3 * N))
    W = (rng.standard_t(3, (K, N)) * 0.02).astype(np.float32)
    W[:, 0] = 0.0
    if N > 2:
        W[:, 1] = 0.0
        W[:4, 1] = np.array([7 / 8, 2.5 / 8, -3.5 / 8, 0.5 / 8], np.float32)
    Wp, sw = q.quantize_weight_int4(torch.from_numpy(W).cuda())
    Wq = q.unpack_int4(Wp)
    torch.cuda.synchronize()
    Wp_o, sw_o = oracle.quantize_weight_int4(W)
    np.testing.assert_array_equal(Wp.cpu().numpy(), Wp_o)
    np.testing.assert_array_equal(to_np(sw).view(np.uint32), sw_o.view(np.uint32))
    np.testing.assert_array_equal(Wq.cpu().numpy(), oracle.unpack_int4(Wp_o))


@pytest.mark.parametrize("M,K,N,r,act", [(1024, 1024, 1024, 8, "bf16"),   # 128x64 tiles
                                          (40, 2048, 1000, 4, "bf16"),    # few tokens
                                          (2304, 2048, 4096, 4, "bf16"),  # forward on CTA pairs
                                          (2100, 1056, 2600, 8, "bf16"),  # CTA pairs, ragged M, N, k-block
                                          (17, 1056, 4096, 8, "f32"),     # few tokens, fp32 outputs
                                          (333, 768, 2304, 4, "bf16"),
                                          (1000, 1312, 264, 8, "bf16"),   # 128x128 tiles
                                          (4096, 768, 768, 4, "bf16"),    # 256x128 tiles
                                          (96, 256, 10, 8, "bf16"),       # CUDA-core dX
                                          (64, 256, 128, 4, "f32"),       # fp32 activations
                                          (200, 800, 264, 16, "bf16"),    # K % 128 == 32: ragged k-block
                                          (850, 4736, 640, 4, "bf16")])   # CTA-pair dX
def test_int4_layer_matches_oracle(q, M, K, N, r, act):
    """An int4 layer: the forward from the packed codes bit-identical to the
    int8 forward on the unpacked codes (accumulator bit-exact against the
    oracle), dX from the packed codes bit-identical to the int8 path and
    within tolerance of the oracle, dA/dB/dbias against the oracle, and the
    int4 merge bit-exact."""
    spec = _edge_spec(M, K, N, r, act=act, seed=5 * M + K)
    d = inputs.layer_inputs(spec)
    from parity import act_torch
    tdt = act_torch(act)
    Wp, sw = q.quantize_weight_int4(torch.from_numpy(d["W"]).cuda())
    Wq8 = q.unpack_int4(Wp)
    layer = q.Layer(Wq=Wq8, sw=sw, bias=torch.from_numpy(d["bias"]).cuda(),
                    A=torch.from_numpy(d["A"]).cuda(), B=torch.from_numpy(d["B"]).cuda(),
                    alpha=spec.alpha, act=tdt)
    D = layer.desc()
    X = torch.from_numpy(d["X"]).to(tdt).cuda()
    dY = torch.from_numpy(d["dY"]).to(tdt).cuda()
    ws = q.workspace(D, M)
    Y, xA, (xq, sx, acc) = q.forward(layer, X, ws, debug=True)
    dB = torch.empty((r, N), device="cuda")
    db = torch.empty((N,), device="cuda")
    q.qlora_lora_grad_dy(D, M, dY, layer.B, xA, dB, db, ws)
    dX4 = torch.full((M, K), float("nan"), dtype=tdt, device="cuda")
    dX8 = torch.empty((M, K), dtype=tdt, device="cuda")
    q.qlora_gemm_dx_int4(D, M, dY, Wp, sw, layer.A, dX4, ws)
    q.qlora_gemm_dx(D, M, dY, Wq8, sw, layer.A, dX8, ws)
    dA = torch.empty((K, r), device="cuda")
    q.qlora_lora_grad_x(D, M, X, dA, ws)
    Wp2, sw2 = q.merge_int4(D, Wp, sw, layer.A, layer.B)
    # the forward from the packed codes, against the int8 forward on the unpacked ones
    Y4 = torch.full_like(Y, float("nan"))
    acc4 = torch.full_like(acc, -1)
    q.qlora_gemm_forward_int4(D, M, xq, sx, Wp, sw, layer.bias, xA, layer.B, Y4, acc4)
    torch.cuda.synchronize()
    assert q.qlora_device_status() == 0
    assert torch.equal(dX4, dX8)
    assert torch.equal(acc4, acc) and torch.equal(Y4, Y)

    Wp_o, sw_o = oracle.quantize_weight_int4(d["W"])
    codes = oracle.unpack_int4(Wp_o)
    rows = np.arange(M) if M <= 1024 else np.unique(np.concatenate(
        [[0, M - 1], np.random.Generator(np.random.PCG64(M)).choice(M, 192, replace=False)]))
    f = oracle.forward(d["X"][rows], codes, sw_o, d["bias"], d["A"], d["B"], spec.alpha)
    np.testing.assert_array_equal(to_np(acc)[rows], f["acc"])
    assert_close(to_np(Y)[rows], f["y"], act, "Y")
    b_rows = oracle.backward(d["X"][rows], d["dY"][rows], codes, sw_o, d["A"], d["B"], spec.alpha,
                             want_dx=True, act=act)
    assert_close(to_np(dX4)[rows], b_rows["dX"], act, "dX (int4)")
    b_full = oracle.backward(d["X"], d["dY"], codes, sw_o, d["A"], d["B"], spec.alpha,
                             want_dx=False, act=act)
    assert_close(to_np(dA), b_full["dA"], act, "dA")
    assert_close(to_np(dB), b_full["dB"], act, "dB")
    assert_close(to_np(db), b_full["dbias"], act, "dbias")
    Wp2_o, sw2_o = oracle.merge_int4(Wp_o, sw_o, d["A"], d["B"], spec.alpha)
    np.testing.assert_array_equal(Wp2.cpu().numpy(), Wp2_o)
    np.testing.assert_array_equal(to_np(sw2).view(np.uint32), sw2_o.view(np.uint32))
