"""The parity checker itself (no GPU): the bf16 tolerance must reject a small
systematic error in outputs of small magnitude, such as the dX of the GPT-2
projections (dY ~ N(0, 1e-2), so |dX| ~ 1e-2, the size of the absolute
tolerance term).  The planted error is applied to the oracle's own result."""
import numpy as np
import pytest

import oracle
from lora_fine_tuning_qlora_b200 import inputs

from parity import assert_close


def _gpt2_small_dx():
    spec = inputs.scaled(inputs.gpt2_base()[0], M=64, N=256)
    d = inputs.layer_inputs(spec)
    Wq, sw = oracle.quantize_weight(d["W"])
    b = oracle.backward(d["X"], d["dY"], Wq, sw, d["A"], d["B"], spec.alpha, want_dx=True,
                        act="bf16")
    return oracle.round_bf16(b["dX"]), b["dX"]


def test_bf16_check_accepts_the_rounded_result():
    got, ref = _gpt2_small_dx()
    assert_close(got, ref, "bf16", "dX rounded to bf16")


@pytest.mark.parametrize("scale", [1.05, 0.95])
def test_bf16_check_rejects_a_5_percent_systematic_error(scale):
    got, ref = _gpt2_small_dx()
    assert np.abs(ref).max() < 0.2  # small outputs: the elementwise atol alone would pass
    with pytest.raises(AssertionError):
        assert_close(got * scale, ref, "bf16", "dX x %.2f" % scale)
