"""GPU parity of the outlier-compensated int8 kernels (keras-llm-light,
"Weights quantization" and "Simplified Int8Variable quantization") against
the CPU oracle: the quantizer bit-exact (codes in both layouts, the affine
parameters and the set of outliers of every bucket), the layer's forward and
backward within the activation dtype's tolerance.  Needs a B200."""
import numpy as np
import pytest
import torch

import oracle
from lora_fine_tuning_qlora_b200 import inputs

from parity import act_torch, assert_close, to_np

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


def _bucket_entries(start, ent, rows, cols):
    """(row, col, fp16 bits) of every stored outlier of one layout."""
    start = start.astype(np.int64)
    nb = (cols + 127) // 128
    assert start.shape == (rows * nb + 1,)
    assert start[0] == 0 and np.all(np.diff(start) >= 0)
    count = int(start[-1])
    e = ent[:count].view(np.uint32).astype(np.int64)
    bucket = np.repeat(np.arange(rows * nb), np.diff(start))
    col = (bucket % nb) * 128 + (e >> 16)
    row = bucket // nb
    assert np.all((e >> 16) < 128) and np.all(col < cols)
    return row, col, (e & 0xFFFF).astype(np.uint16)


def _check_quantizer(qk, W):
    K, N = W.shape
    ref = oracle.quantize_outlier_int8(W)
    codes_kn = to_np(qk.codes_kn)
    codes_nk = to_np(qk.codes_nk)
    np.testing.assert_array_equal(codes_kn, ref["codes"])
    np.testing.assert_array_equal(codes_nk, ref["codes"].T)
    par = to_np(qk.par)
    want = np.array([ref["lo"], ref["hi"], ref["scale"], ref["bias"]], np.float32)
    np.testing.assert_array_equal(par, want)
    assert qk.count == ref["count"] <= q_cap(K, N)
    # the outliers, as sets of (k, n, fp16 bits), in both layouts
    ks, ns = np.nonzero(ref["is_outlier"])
    bits = ref["values"][ks, ns].astype(np.float16).view(np.uint16)
    want_set = sorted(zip(ks.tolist(), ns.tolist(), bits.tolist()))
    n_, k_, b_ = _bucket_entries(to_np(qk.start_nk), to_np(qk.ent_nk), N, K)
    assert sorted(zip(k_.tolist(), n_.tolist(), b_.tolist())) == want_set
    k2, n2, b2 = _bucket_entries(to_np(qk.start_kn), to_np(qk.ent_kn), K, N)
    assert sorted(zip(k2.tolist(), n2.tolist(), b2.tolist())) == want_set
    return ref


def q_cap(K, N):
    from lora_fine_tuning_qlora_b200 import qlora
    return qlora.qlora_outlier_cap(K, N)


# ---------------------------------------------------------------- quantizer
@pytest.mark.parametrize("K,N,dist", [(768, 2304, "normal002_outliers"),
                                      (3072, 768, "normal002_outliers"),
                                      (1000, 10, "normal002_outliers"),
                                      (100, 130, "student_t3"),
                                      (4096, 4096, "student_t3"),
                                      (16, 1, "glorot")])
def test_outlier_quantizer_bit_exact(q, K, N, dist):
    spec = inputs.LayerSpec("w", M=1, K=K, N=N, r=1, alpha=1.0, w_dist=dist, seed=K + N)
    W = inputs.layer_inputs(spec, with_x=False, with_dy=False)["W"]
    qk = q.quantize_outlier(torch.from_numpy(W).cuda())
    torch.cuda.synchronize()
    _check_quantizer(qk, W)


def test_outlier_quantizer_ties_and_constant_kernels(q):
    """Cutoffs that fall on repeated entries (ties across the order
    statistics), and a constant kernel (scale 0: every code 0, no outliers)."""
    rng = np.random.Generator(np.random.PCG64(5))
    W = rng.integers(-3, 4, size=(64, 96)).astype(np.float32) * np.float32(0.25)
    W[0, :5] = [9.0, -9.0, 8.0, -7.5, 6.25]
    qk = q.quantize_outlier(torch.from_numpy(W).cuda())
    torch.cuda.synchronize()
    _check_quantizer(qk, W)
    C = np.full((32, 48), -0.375, np.float32)
    qc = q.quantize_outlier(torch.from_numpy(C).cuda())
    torch.cuda.synchronize()
    ref = _check_quantizer(qc, C)
    assert ref["count"] == 0 and ref["scale"] == 0.0


def test_outlier_quantizer_rejects_small_capacity(q):
    W = torch.zeros((64, 64), dtype=torch.float32, device="cuda")
    qk = q.outlier_kernel_buffers(64, 64)
    qk.ent_nk = qk.ent_nk[:1]
    qk.ent_kn = qk.ent_kn[:1]
    ws = torch.empty(q.qlora_outlier_workspace_bytes(64, 64), dtype=torch.uint8, device="cuda")
    if q.qlora_outlier_cap(64, 64) > 1:
        with pytest.raises(q.QLoraError) as e:
            q.qlora_outlier_quantize(W, qk, ws)
        assert e.value.code == -1


# ---------------------------------------------------------------- the layer
def _run_layer(q, spec):
    d = inputs.layer_inputs(spec)
    M, K, N, r = spec.M, spec.K, spec.N, spec.r
    act = spec.act
    tdt = act_torch(act)
    qk = q.quantize_outlier(torch.from_numpy(d["W"]).cuda())
    X = torch.from_numpy(d["X"]).to(tdt).cuda()
    dY = torch.from_numpy(d["dY"]).to(tdt).cuda()
    A = torch.from_numpy(d["A"]).cuda()
    B = torch.from_numpy(d["B"]).cuda()
    bias = torch.from_numpy(d["bias"]).cuda() if d["bias"] is not None else None
    desc = q.desc(K, N, r, spec.alpha, tdt)
    ws = q.workspace(desc, M)
    Y = torch.empty((M, N), dtype=tdt, device="cuda")
    xA = torch.empty((M, r), dtype=torch.float32, device="cuda")
    q.qlora_outlier_forward(desc, M, X, qk, bias, A, B, Y, xA, ws)
    dX = torch.empty((M, K), dtype=tdt, device="cuda")
    dA = torch.empty((K, r), dtype=torch.float32, device="cuda")
    dB = torch.empty((r, N), dtype=torch.float32, device="cuda")
    dbias = torch.empty((N,), dtype=torch.float32, device="cuda")
    q.qlora_outlier_backward(desc, M, X, dY, qk, A, B, xA, dX, dA, dB, dbias, ws)
    torch.cuda.synchronize()
    assert q.qlora_device_status() == 0
    ref = _check_quantizer(qk, d["W"])
    f = oracle.forward_outlier(d["X"], ref, d["bias"], d["A"], d["B"], spec.alpha, act)
    b = oracle.backward_outlier(d["X"], d["dY"], ref, d["A"], d["B"], spec.alpha, act)
    assert_close(to_np(xA), f["xA"], act, "xA")
    assert_close(to_np(Y), f["y"], act, "Y")
    assert_close(to_np(dX), b["dX"], act, "dX")
    assert_close(to_np(dA), b["dA"], act, "dA")
    assert_close(to_np(dB), b["dB"], act, "dB")
    assert_close(to_np(dbias), b["dbias"], act, "dbias")


@pytest.mark.parametrize("i", range(4))
def test_outlier_gpt2_layers(q, i):
    """The four GPT-2 base Dense shapes (0.1% of the weights x20), 300 tokens."""
    _run_layer(q, inputs.scaled(inputs.gpt2_base()[i], M=300))


@pytest.mark.parametrize("i", [2, 3])
def test_outlier_gpt2_layers_on_cta_pairs(q, i):
    """2560 tokens: the 768 -> 3072 forward and the 3072 -> 768 backward GEMMs
    run on CTA pairs (256 x 256 tiles), the other direction on single CTAs."""
    _run_layer(q, inputs.scaled(inputs.gpt2_base()[i], M=2560))


@pytest.mark.parametrize("M,K,N,r,act,bias", [
    (130, 256, 200, 8, "f32", "normal001"),     # fp32 activations: CUDA-core path
    (97, 784, 520, 16, "bf16", "none"),         # N % 16 == 8: forward on CUDA cores, no bias
    (70, 128, 48, 64, "bf16", "normal001"),     # rank 64: rank-r epilogue on CUDA cores
    (1000, 1088, 4752, 8, "bf16", "normal001"),  # forward on CTA pairs, ragged M, N tiles
    (1, 64, 16, 1, "bf16", "normal001"),        # one token
])
def test_outlier_layer_shapes(q, M, K, N, r, act, bias):
    spec = inputs.LayerSpec("outlier", M=M, K=K, N=N, r=r, alpha=2.0 * r, act=act,
                            x_dist="normal", w_dist="normal002_outliers", a_dist="he_uniform",
                            b_std=0.01, bias_dist=bias, dy_std=1e-2, seed=M + K + N + r)
    _run_layer(q, spec)


def test_outlier_layer_empty_batch(q):
    """M == 0: nothing to compute; the parameter gradients are zero."""
    K, N, r = 64, 32, 4
    qk = q.quantize_outlier(torch.randn(K, N, device="cuda") * 0.02)
    desc = q.desc(K, N, r, 4.0, torch.bfloat16)
    ws = q.workspace(desc, 0)
    # non-empty stand-ins: a 0-row tensor has no device address to pass
    X = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    dY = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    A = torch.randn(K, r, device="cuda")
    B = torch.randn(r, N, device="cuda")
    xA = torch.empty(4, device="cuda")
    Y = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    q.qlora_outlier_forward(desc, 0, X, qk, None, A, B, Y, xA, ws)
    dA = torch.full((K, r), 7.0, device="cuda")
    dB = torch.full((r, N), 7.0, device="cuda")
    db = torch.full((N,), 7.0, device="cuda")
    q.qlora_outlier_backward(desc, 0, X, dY, qk, A, B, xA, None, dA, dB, db, ws)
    torch.cuda.synchronize()
    assert float(dA.abs().max()) == 0 and float(dB.abs().max()) == 0 and float(db.abs().max()) == 0
