"""Failure detection on the GPU without a fault: a bounded wait that runs out
(on a barrier nothing arrives on) is reported through the status word, the
report is cleared once read, and the context keeps working."""

import math

import pytest
import torch

from oracle import attention_forward
from parity import assert_close, f64, run_fwd
from sqa_inputs import attention_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sqa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_query_attention_b200 as lib
    return lib


def test_bounded_wait_timeout_is_reported_and_cleared(sqa):
    sqa.sqa_device_status()  # start from a clean status word
    sqa.sqa_selftest_wait_timeout(50)
    with pytest.raises(sqa.SQAError) as err:
        sqa.sqa_device_status()
    assert err.value.status == sqa.SQA_ERR_TIMEOUT
    sqa.sqa_device_status()  # read once: cleared

    # The context still runs the real kernels correctly.
    x = attention_inputs(1, 300, 8, 4, 64, seed=55, device="cuda")
    o, lse = run_fwd(sqa, x["q"], x["k"], x["v"], True)
    sqa.sqa_device_status()
    o_ref, lse_ref = attention_forward(f64(x["q"]), f64(x["k"]), f64(x["v"]), True, 1 / math.sqrt(64))
    assert_close(f64(o), o_ref, "O after a reported timeout")
    assert_close(f64(lse), lse_ref, "LSE after a reported timeout")
