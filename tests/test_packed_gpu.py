"""GPU parity of the attention core on a packed QKV buffer
[B, N, H_q + 2 H_kv, d] (the output of one fused input projection): forward
and gradient against the fp64 oracle, and bitwise equality with the dense
entry points on the same bits."""

import math

import pytest
import torch

from oracle import attention_backward, attention_forward
from parity import assert_close, assert_close_scaled, f64, run_bwd, run_fwd
from sqa_inputs import attention_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sqa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_query_attention_b200 as lib
    return lib


@pytest.mark.parametrize("B,N,H_q,H_kv,d,causal", [
    (2, 256, 4, 2, 32, True),
    (1, 1000, 8, 4, 64, True),
    (2, 300, 8, 8, 128, False),
    (1, 513, 4, 1, 16, True),
    (3, 129, 6, 2, 64, False),
    # Non-causal with few key tiles / query tiles: dK/dV split over clusters
    # (d = 64), and the forward, dK/dV and dQ splits (d = 128), all writing
    # through the packed strides.
    (1, 2048, 8, 4, 64, False),
    (1, 2048, 4, 4, 128, False),
])
def test_packed_matches_oracle_and_dense(sqa, B, N, H_q, H_kv, d, causal):
    x = attention_inputs(B, N, H_q, H_kv, d, seed=400 + N, with_dout=True, device="cuda")
    qkv = torch.cat([x["q"], x["k"], x["v"]], dim=2).contiguous()
    scale = 1 / math.sqrt(d)
    o = torch.empty((B, N, H_q, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, H_q, N), dtype=torch.float32, device="cuda")
    sqa.sqa_attn_fwd_packed(qkv, o, sqa.SQA_DT_F32, lse, B, N, H_q, H_kv, d, causal, scale)
    dqkv = torch.empty((B, N, H_q + 2 * H_kv, d), dtype=torch.float32, device="cuda")
    wsb = sqa.sqa_attn_bwd_workspace_size(B, N, H_q, H_kv, d)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    sqa.sqa_attn_bwd_packed(qkv, o, sqa.SQA_DT_F32, x["do"], lse, dqkv, sqa.SQA_DT_F32, B, N, H_q, H_kv, d,
                            causal, scale, ws, wsb)
    o2, lse2 = run_fwd(sqa, x["q"], x["k"], x["v"], causal)
    dq2, dk2, dv2 = run_bwd(sqa, x["q"], x["k"], x["v"], o2, x["do"], lse2, causal)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    dq, dk, dv = dqkv[:, :, :H_q], dqkv[:, :, H_q:H_q + H_kv], dqkv[:, :, H_q + H_kv:]
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    assert torch.equal(dq, dq2) and torch.equal(dk, dk2) and torch.equal(dv, dv2)
    ro, rl = attention_forward(f64(x["q"]), f64(x["k"]), f64(x["v"]), causal, scale)
    rq, rk, rv = attention_backward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["do"]), causal, scale)
    assert_close(f64(o), ro, "O")
    assert_close(f64(lse), rl, "LSE")
    assert_close(f64(dq), rq, "dQ")
    assert_close(f64(dk), rk, "dK")
    assert_close(f64(dv), rv, "dV")


def test_packed_bf16_gradients_fill_the_whole_buffer(sqa):
    """Every entry of dQKV is written: a buffer pre-filled with NaN comes back
    finite."""
    B, N, H_q, H_kv, d = 2, 200, 8, 2, 64
    x = attention_inputs(B, N, H_q, H_kv, d, seed=77, with_dout=True, device="cuda")
    qkv = torch.cat([x["q"], x["k"], x["v"]], dim=2).contiguous()
    o = torch.empty((B, N, H_q, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H_q, N), dtype=torch.float32, device="cuda")
    sqa.sqa_attn_fwd_packed(qkv, o, sqa.SQA_DT_BF16, lse, B, N, H_q, H_kv, d, True, 0.125)
    dqkv = torch.full((B, N, H_q + 2 * H_kv, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    wsb = sqa.sqa_attn_bwd_workspace_size(B, N, H_q, H_kv, d)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    sqa.sqa_attn_bwd_packed(qkv, o, sqa.SQA_DT_BF16, x["do"], lse, dqkv, sqa.SQA_DT_BF16, B, N, H_q, H_kv, d,
                            True, 0.125, ws, wsb)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    assert torch.isfinite(dqkv.float()).all()
    rq, rk, rv = attention_backward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["do"]), True, 0.125)
    # bf16 gradients: dV of the first keys sums P dO over up to N rows and 4
    # heads and reaches |dV| ~ 8-16, where one bf16 rounding alone is up to
    # 2^-9 * 16 = 0.031; for dK and dV the bound is therefore taken relative
    # to the tensor's scale (max|err| <= 2e-2 * max(1, max|ref|), relL2 <=
    # 1e-2).  dQ stays near unit size and takes the plain bound.
    assert_close(f64(dqkv[:, :, :H_q]), rq, "dQ")
    assert_close_scaled(f64(dqkv[:, :, H_q:H_q + H_kv]), rk, "dK")
    assert_close_scaled(f64(dqkv[:, :, H_q + H_kv:]), rv, "dV")
