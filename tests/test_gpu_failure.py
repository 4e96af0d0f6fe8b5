"""Failure detection on the GPU without a fault: a kernel's bounded wait runs
out (a barrier that nothing signals), the kernel records a timeout in the
device status word and exits; the host reads QLORA_ETIMEOUT and the context
stays usable for the next layer call."""
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


def test_bounded_wait_reports_timeout_and_context_survives(q):
    assert q.qlora_device_status() == 0
    q.qlora_selftest_wait_timeout(2000)          # gives up after 2 ms
    assert q.qlora_device_status() == -6         # QLORA_ETIMEOUT, then cleared
    assert q.qlora_device_status() == 0
    # the context still runs a layer
    from lora_fine_tuning_qlora_b200 import inputs
    import sys, os
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    from parity import run_and_compare
    spec = inputs.LayerSpec("after_timeout", M=64, K=128, N=96, r=4, alpha=4.0, act="bf16", seed=9)
    run_and_compare(spec, q)


def test_selftest_rejects_bad_limit(q):
    with pytest.raises(q.QLoraError):
        q.qlora_selftest_wait_timeout(0)
