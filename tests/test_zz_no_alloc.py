"""qlora_backward_noalloc: the backward with the library's static scratch in
place of a caller-supplied workspace.  Both entry points run the same
deterministic kernels in the same order, so two calls in a row through the C
ABI must each give results bit-identical to qlora_backward (the workspace
entry point) on the same inputs, even after a call on a larger layer with
other inputs has left different data in the shared scratch; one case is also
checked against the CPU oracle within the parity tolerance.

Collected last on purpose: it must also pass after every other test has run
in the same process, as well as alone in a fresh one."""
import ctypes

import pytest
import torch

from lora_fine_tuning_qlora_b200 import inputs

import oracle
from parity import act_torch, assert_close, device_layer, to_np


@pytest.fixture(scope="module")
def q():
    from lora_fine_tuning_qlora_b200 import build
    build.build()
    from lora_fine_tuning_qlora_b200 import qlora
    return qlora


def _grads(q, layer, M, dev, want_dbias):
    dX = torch.full((M, layer.K), float("nan"), dtype=layer.act, device=dev)
    dA = torch.full((layer.K, layer.r), float("nan"), device=dev)
    dB = torch.full((layer.r, layer.N), float("nan"), device=dev)
    dbias = torch.full((layer.N,), float("nan"), device=dev) if want_dbias else None
    return dX, dA, dB, dbias


SPECS = [
    inputs.mlp_stack()[1],                             # bf16 1024x1024, r 8
    inputs.single_fp32(),                              # fp32 64x784x128, r 4
    inputs.scaled(inputs.gpt2_base()[0], M=333),       # bf16 ragged M, N = 2304
]


@pytest.mark.gpu
@pytest.mark.parametrize("spec", SPECS, ids=lambda s: s.name)
def test_noalloc_backward_matches_workspace_backward(q, spec):
    if not torch.cuda.is_available():
        pytest.fail("this test needs a CUDA device")
    dev = torch.device("cuda", 0)
    d = inputs.layer_inputs(spec)
    layer = device_layer(spec, d, q)
    tdt = act_torch(spec.act)
    X = torch.from_numpy(d["X"]).to(tdt).to(dev)
    dY = torch.from_numpy(d["dY"]).to(tdt).to(dev)
    M = spec.M
    D = layer.desc()
    ws = q.workspace(D, M, dev)
    _, xA = q.forward(layer, X, ws)
    want_dbias = layer.bias is not None

    # first fill the shared scratch with another layer's data: more rows and
    # more G slices than the layer under test, other inputs
    big = inputs.scaled(spec, M=spec.M + 77, N=spec.N + 136 if spec.N % 8 == 0 else spec.N,
                        seed=spec.seed + 17)
    db = inputs.layer_inputs(big)
    lb = device_layer(big, db, q)
    Xb = torch.from_numpy(db["X"]).to(tdt).to(dev)
    dYb = torch.from_numpy(db["dY"]).to(tdt).to(dev)
    wsb = q.workspace(lb.desc(), big.M, dev)
    _, xAb = q.forward(lb, Xb, wsb)
    q.qlora_backward_noalloc(lb.desc(), big.M, Xb, dYb, lb.Wq, lb.sw, lb.A, lb.B, xAb,
                             *_grads(q, lb, big.M, dev, lb.bias is not None))

    # two scratch-free calls in a row, each into fresh outputs
    runs = []
    for _ in range(2):
        out = _grads(q, layer, M, dev, want_dbias)
        q.qlora_backward_noalloc(D, M, X, dY, layer.Wq, layer.sw, layer.A, layer.B, xA, *out)
        runs.append(out)
    torch.cuda.synchronize()
    assert q.qlora_device_status() == 0

    # the workspace entry point on the same inputs
    ref = _grads(q, layer, M, dev, want_dbias)
    q.qlora_backward(D, M, X, dY, layer.Wq, layer.sw, layer.A, layer.B, xA, *ref, ws)
    torch.cuda.synchronize()
    assert q.qlora_device_status() == 0

    names = ("dX", "dA", "dB", "dbias")
    for i, out in enumerate(runs):
        for name, g, r in zip(names, out, ref):
            if r is None:
                continue
            assert torch.equal(g, r), "call %d %s differs from qlora_backward" % (i + 1, name)

    # and the second call against the oracle
    Wq_o, sw_o = oracle.quantize_weight(d["W"])
    b = oracle.backward(d["X"], d["dY"], Wq_o, sw_o, d["A"], d["B"], spec.alpha, want_dx=True,
                        act=spec.act)
    for name, g in zip(names, runs[1]):
        if g is None:
            continue
        act = spec.act if name == "dX" else ("f32" if spec.act == "f32" else "bf16")
        assert_close(to_np(g), b[name], act, "oracle vs call 2 %s" % name)


def test_noalloc_rejects_layers_above_the_static_scratch(q):
    """A bf16 layer with N = 4096, r = 64, M = 1024 has 32 slices of G
    (32 * 1024 * 64 * 4 = 8 MiB) plus G itself (256 KiB): 8650752 bytes, more
    than the static scratch, so it is refused before anything is launched
    (fake, aligned pointers; no GPU needed)."""
    P = ctypes.c_void_p
    d = q.desc(1024, 4096, 64, 64.0, torch.bfloat16)
    ptrs = [P(0x10000 * (i + 1)) for i in range(11)]
    rc = q.lib().qlora_backward_noalloc(ctypes.byref(d), 1024, *ptrs, None)
    assert rc == -3
    msg = q.lib().qlora_last_error()
    assert b"static scratch" in msg and b"8650752" in msg and b"8388608" in msg
