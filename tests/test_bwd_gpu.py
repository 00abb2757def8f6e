"""GPU parity of the SQA attention-core gradient against the fp64 oracle."""

import math

import pytest
import torch

from oracle import attention_backward
from parity import assert_close, f64, run_bwd, run_fwd
from sqa_inputs import attention_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sqa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_query_attention_b200 as lib
    return lib


def _check_bwd(sqa, B, N, H_q, H_kv, d, causal, seed, o_dtype=torch.float32, grad_dtype=torch.float32):
    x = attention_inputs(B, N, H_q, H_kv, d, seed, with_dout=True, device="cuda")
    o, lse = run_fwd(sqa, x["q"], x["k"], x["v"], causal, out_dtype=o_dtype)
    dq, dk, dv = run_bwd(sqa, x["q"], x["k"], x["v"], o, x["do"], lse, causal, grad_dtype=grad_dtype)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    rq, rk, rv = attention_backward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["do"]), causal, 1 / math.sqrt(d))
    assert_close(f64(dq), rq, "dQ")
    assert_close(f64(dk), rk, "dK")
    assert_close(f64(dv), rv, "dV")


def test_training_step_config(sqa):
    """B=4, N=8192, H_q=8, H_kv=4, d=64, causal, seed 4: dQ, and dK/dV summed
    over each KV head's two query heads."""
    _check_bwd(sqa, 4, 8192, 8, 4, 64, True, seed=4)


@pytest.mark.parametrize("B,N,H_q,H_kv,d,causal", [
    (1, 1, 2, 1, 64, True),
    (2, 127, 4, 2, 64, True),
    (1, 129, 8, 2, 128, False),
    (3, 200, 4, 4, 32, True),
    (1, 256, 16, 1, 16, False),
    (1, 383, 8, 4, 64, False),
    (2, 520, 2, 1, 128, True),
    (1, 1000, 8, 8, 64, True),
])
def test_bwd_shape_sweep(sqa, B, N, H_q, H_kv, d, causal):
    _check_bwd(sqa, B, N, H_q, H_kv, d, causal, seed=2000 + N)


@pytest.mark.parametrize("H_q,H_kv,d,causal", [(6, 2, 64, True), (12, 4, 32, False), (6, 1, 128, True)])
def test_bwd_group_not_power_of_two(sqa, H_q, H_kv, d, causal):
    """G = 3 or 6: dK/dV sum over all G heads of the group; dQ tiles pack the
    largest power of two dividing G."""
    _check_bwd(sqa, 1, 300, H_q, H_kv, d, causal, seed=70 + H_q)


def test_bwd_bf16_io(sqa):
    _check_bwd(sqa, 2, 384, 8, 4, 64, True, seed=21, o_dtype=torch.bfloat16, grad_dtype=torch.bfloat16)


@pytest.mark.parametrize("H_q,H_kv,causal", [(32, 1, True), (128, 1, False), (64, 2, True)])
def test_bwd_wide_groups(sqa, H_q, H_kv, causal):
    """dK/dV summed over up to 128 query heads of one KV head; dQ tiles of
    128 / G tokens.  dK and dV grow with the G-fold group sum (|dV| of the
    first keys reaches ~10-20 here) while bf16 P and dS contribute a relative
    error per term, so the absolute bound scales with the tensor
    (tests/parity.py assert_close_scaled); the relative L2 bound is the
    usual 1e-2."""
    from parity import assert_close_scaled
    B, N, d = 1, 150, 64
    x = attention_inputs(B, N, H_q, H_kv, d, 300 + H_q, with_dout=True, device="cuda")
    o, lse = run_fwd(sqa, x["q"], x["k"], x["v"], causal)
    dq, dk, dv = run_bwd(sqa, x["q"], x["k"], x["v"], o, x["do"], lse, causal)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    rq, rk, rv = attention_backward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["do"]), causal, 1 / math.sqrt(d))
    assert_close(f64(dq), rq, "dQ")
    assert_close_scaled(f64(dk), rk, "dK")
    assert_close_scaled(f64(dv), rv, "dV")
