"""The replayable layer step (lora_fine_tuning_qlora_b200.step.LayerStep):
its five launch groups, with the X pass on a second stream beside the dX
GEMM and captured into a CUDA graph, give bit for bit what the composite
qlora_forward / qlora_backward calls give on the same inputs (the same
deterministic kernels), eagerly and on graph replay.  Needs a B200."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.fail("these tests need a CUDA device")
    from lora_fine_tuning_qlora_b200 import build
    build.build()
    from lora_fine_tuning_qlora_b200 import qlora
    return qlora


def _layer(q, K, N, r, act, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    W = torch.randn((K, N), generator=g) * 0.05
    Wq, sw = q.quantize_weight(W.cuda())
    return q.Layer(Wq=Wq, sw=sw, bias=(torch.randn(N, generator=g) * 0.1).cuda(),
                   A=(torch.randn(K, r, generator=g) * 0.05).cuda(),
                   B=(torch.randn(r, N, generator=g) * 0.05).cuda(), alpha=2.0 * r, act=act)


@pytest.mark.parametrize("M,K,N,r,act", [
    (16, 4096, 4096, 4, torch.bfloat16),    # few tokens: the GEMMs leave most SMs to the X pass
    (2304, 1024, 2048, 8, torch.bfloat16),  # CTA-pair GEMMs with a partial last wave
    (300, 784, 520, 4, torch.float32),      # fp32 activations, ragged tiles
    (640, 256, 384, 4, torch.float32),      # fp32 with the second stream (from 512 tokens)
])
def test_step_matches_composite_calls(q, M, K, N, r, act):
    from lora_fine_tuning_qlora_b200 import step
    layer = _layer(q, K, N, r, act, M + K + N)
    g = torch.Generator(device="cpu").manual_seed(M)
    X = torch.randn((M, K), generator=g).to(act).cuda()
    dY = (torch.randn((M, N), generator=g) * 0.01).to(act).cuda()

    ws = q.workspace(layer.desc(), M, torch.device("cuda"))
    Y, xA = q.forward(layer, X, ws)
    dX, dA, dB, dbias = q.backward(layer, X, dY, xA, ws)
    torch.cuda.synchronize()

    for overlap in (True, False):
        st = step.LayerStep(layer, M, "cuda", overlap_x=overlap)
        st.X.copy_(X)
        st.dY.copy_(dY)
        st.run()
        torch.cuda.synchronize()
        for name, a, b in (("Y", st.Y, Y), ("xA", st.xA, xA), ("dX", st.dX, dX), ("dA", st.dA, dA),
                           ("dB", st.dB, dB), ("dbias", st.dbias, dbias)):
            assert torch.equal(a, b), ("eager", overlap, name)
        # graph replay after the outputs are cleared
        st.capture(warmup=1)
        for t in (st.Y, st.dX, st.grad_flat):
            t.fill_(float("nan"))
        st.replay()
        torch.cuda.synchronize()
        for name, a, b in (("Y", st.Y, Y), ("dX", st.dX, dX), ("dA", st.dA, dA), ("dB", st.dB, dB),
                           ("dbias", st.dbias, dbias)):
            assert torch.equal(a, b), ("replay", overlap, name)
        assert np.isfinite(st.grad_flat.cpu().numpy()).all()


def test_composite_backward_in_a_graph(q):
    """qlora_backward with its second stream (from 512 tokens) captured into
    a CUDA graph and replayed gives what the eager call gives."""
    M, K, N, r, act = 1024, 1024, 1536, 4, torch.bfloat16
    layer = _layer(q, K, N, r, act, 5)
    g = torch.Generator(device="cpu").manual_seed(6)
    X = torch.randn((M, K), generator=g).to(act).cuda()
    dY = (torch.randn((M, N), generator=g) * 0.01).to(act).cuda()
    ws = q.workspace(layer.desc(), M, torch.device("cuda"))
    Y, xA = q.forward(layer, X, ws)
    ref = q.backward(layer, X, dY, xA, ws)  # eager: also creates the second stream
    torch.cuda.synchronize()
    outs = [torch.empty_like(t) for t in ref]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        q.qlora_backward(layer.desc(), M, X, dY, layer.Wq, layer.sw, layer.A, layer.B, xA,
                         outs[0], outs[1], outs[2], outs[3], ws, s)
    for t in outs:
        t.fill_(float("nan"))
    graph.replay()
    torch.cuda.synchronize()
    for name, a, b in zip(("dX", "dA", "dB", "dbias"), outs, ref):
        assert torch.equal(a, b), name
