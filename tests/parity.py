"""Shared helpers of the GPU parity tests: run one layer through the C ABI
and through the CPU oracle on the same seeded inputs, and compare.

Tolerances (stated in the layer's own terms):
  * int8 codes, int32 accumulators, row/channel scales, merged kernels:
    bit-exact;
  * fp32 activations: norm-wise max relative error
    max|gpu - ref| / max|ref| <= 1e-5;
  * bf16 activations (and the fp32 gradients of a bf16 layer): elementwise
    |gpu - ref| <= 1e-2 + 2e-2 * |ref|, against the fp64 oracle, and, so that
    the absolute term cannot hide an error in outputs of small magnitude
    (dY ~ N(0, 1e-2) gives |dX| ~ 1e-2), also norm-wise
    max|gpu - ref| <= 1e-2 * max|ref|: a 5% systematic error fails it.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from lora_fine_tuning_qlora_b200 import inputs

F32_RTOL = 1e-5
BF16_RTOL = 2e-2
BF16_ATOL = 1e-2
BF16_NORM = 1e-2


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach()
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.cpu().numpy()


def assert_close(gpu, ref, act: str, what: str, norm: bool = True):
    g = np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), what + ": non-finite values"
    if act == "f32":
        scale = np.abs(r).max()
        err = np.abs(g - r).max()
        assert err <= F32_RTOL * max(scale, 1e-30), "%s: max rel err %.3g" % (what, err / max(scale, 1e-30))
    else:
        bad = np.abs(g - r) > BF16_ATOL + BF16_RTOL * np.abs(r)
        if bad.any():
            i = np.argwhere(bad)[0]
            raise AssertionError("%s: %d elements out of tolerance, first at %s: gpu %r ref %r"
                                 % (what, int(bad.sum()), tuple(i), g[tuple(i)], r[tuple(i)]))
        scale = np.abs(r).max() if r.size else 0.0
        if norm and scale > 0:
            err = np.abs(g - r).max()
            assert err <= BF16_NORM * scale, "%s: norm-wise rel err %.3g" % (what, err / scale)


def act_torch(act: str):
    return torch.bfloat16 if act == "bf16" else torch.float32


def device_layer(spec: inputs.LayerSpec, d, q):
    """Quantizes W on the GPU and returns (Layer, Wq_gpu, sw_gpu)."""
    W = torch.from_numpy(d["W"]).cuda()
    Wq, sw = q.quantize_weight(W)
    bias = torch.from_numpy(d["bias"]).cuda() if d["bias"] is not None else None
    layer = q.Layer(Wq=Wq, sw=sw, bias=bias, A=torch.from_numpy(d["A"]).cuda(),
                    B=torch.from_numpy(d["B"]).cuda(), alpha=spec.alpha, act=act_torch(spec.act))
    return layer


def run_and_compare(spec: inputs.LayerSpec, q, sample_rows=None, check_merge=True, seed=0):
    """Full forward/backward/merge parity of one layer.

    sample_rows: None compares every row; an int n compares Y and dX on n
    seeded row samples (the rows are independent), while dA, dB, dbias are
    always compared in full.
    """
    d = inputs.layer_inputs(spec)
    M, K, N = spec.M, spec.K, spec.N
    act = spec.act
    layer = device_layer(spec, d, q)
    Wq_o, sw_o = oracle.quantize_weight(d["W"])
    np.testing.assert_array_equal(to_np(layer.Wq), Wq_o)
    np.testing.assert_array_equal(to_np(layer.sw).view(np.uint32), sw_o.view(np.uint32))

    tdt = act_torch(act)
    X = torch.from_numpy(d["X"]).to(tdt).cuda()
    dY = torch.from_numpy(d["dY"]).to(tdt).cuda()
    ws = q.workspace(layer.desc(), M)
    Y, xA, (xq, sx, acc) = q.forward(layer, X, ws, debug=True)
    dX, dA, dB, dbias = q.backward(layer, X, dY, xA, ws)
    torch.cuda.synchronize()
    assert q.qlora_device_status() == 0

    if sample_rows is None:
        rows = np.arange(M)
    else:
        rng = np.random.Generator(np.random.PCG64(1000 + seed))
        rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, min(sample_rows, M), replace=False)]))
    Xs = d["X"][rows]
    f = oracle.forward(Xs, Wq_o, sw_o, d["bias"], d["A"], d["B"], spec.alpha)
    np.testing.assert_array_equal(to_np(xq)[rows], f["xq"])
    np.testing.assert_array_equal(to_np(sx)[rows].view(np.uint32), f["sx"].view(np.uint32))
    np.testing.assert_array_equal(to_np(acc)[rows], f["acc"])
    assert_close(to_np(xA)[rows], f["xA"], act, "xA")
    assert_close(to_np(Y)[rows], f["y"], act, "Y")

    b_rows = oracle.backward(Xs, d["dY"][rows], Wq_o, sw_o, d["A"], d["B"], spec.alpha,
                             want_dx=True, act=act)
    assert_close(to_np(dX)[rows], b_rows["dX"], act, "dX")
    if sample_rows is None:
        b_full = b_rows
    else:
        b_full = oracle.backward(d["X"], d["dY"], Wq_o, sw_o, d["A"], d["B"], spec.alpha,
                                 want_dx=False, act=act)
    assert_close(to_np(dA), b_full["dA"], act, "dA")
    assert_close(to_np(dB), b_full["dB"], act, "dB")
    assert_close(to_np(dbias), b_full["dbias"], act, "dbias")

    if check_merge:
        Wq2, sw2 = q.merge(layer)
        Wq2_o, sw2_o = oracle.merge(Wq_o, sw_o, d["A"], d["B"], spec.alpha)
        np.testing.assert_array_equal(to_np(Wq2), Wq2_o)
        np.testing.assert_array_equal(to_np(sw2).view(np.uint32), sw2_o.view(np.uint32))
    return {"layer": layer, "Y": Y, "dX": dX, "dA": dA, "dB": dB}
