"""GPU parity of sliding-window SQA (query t sees keys t - left .. t + right)
against the fp64 oracle: forward output and log-sum-exp, and the gradient.
Windows narrower than a tile, wider than several tiles, one-sided (causal
windows) and two-sided, degenerate ones, and the causal mask as the window
(N, 0)."""

import math

import pytest
import torch

from oracle import attention_backward, attention_forward
from parity import assert_close, f64, run_fwd
from sqa_inputs import attention_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sqa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_query_attention_b200 as lib
    return lib


def _fwd(sqa, x, left, right, out_dtype=torch.float32):
    B, N, H_q, d = x["q"].shape
    H_kv = x["k"].shape[2]
    out = torch.empty((B, N, H_q, d), dtype=out_dtype, device="cuda")
    lse = torch.empty((B, H_q, N), dtype=torch.float32, device="cuda")
    dt = sqa.SQA_DT_BF16 if out_dtype == torch.bfloat16 else sqa.SQA_DT_F32
    sqa.sqa_attn_fwd_window(x["q"], x["k"], x["v"], out, dt, lse, B, N, H_q, H_kv, d, left, right,
                            1 / math.sqrt(d))
    return out, lse


def _bwd(sqa, x, o, lse, left, right):
    B, N, H_q, d = x["q"].shape
    H_kv = x["k"].shape[2]
    dq, dk, dv = (torch.empty(t.shape, dtype=torch.float32, device="cuda") for t in (x["q"], x["k"], x["v"]))
    wsb = sqa.sqa_attn_bwd_workspace_size(B, N, H_q, H_kv, d)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    od = sqa.SQA_DT_BF16 if o.dtype == torch.bfloat16 else sqa.SQA_DT_F32
    sqa.sqa_attn_bwd_window(x["q"], x["k"], x["v"], o, od, x["do"], lse, dq, dk, dv, sqa.SQA_DT_F32, B, N, H_q,
                            H_kv, d, left, right, 1 / math.sqrt(d), ws, wsb)
    return dq, dk, dv


SHAPES = [
    # B, N, H_q, H_kv, d, left, right
    (1, 1000, 8, 4, 64, 127, 0),     # causal window of 128 keys
    (2, 700, 4, 2, 128, 200, 200),   # symmetric local window
    (1, 513, 8, 2, 32, 0, 0),        # each token sees only itself
    (1, 2048, 8, 4, 64, 300, 50),    # lopsided, spans several tiles
    (1, 777, 6, 2, 64, 64, 64),      # G = 3
    (3, 129, 4, 1, 16, 5, 2),        # narrow window, ragged tail
    (1, 300, 16, 4, 128, 1000, 1000),  # sides past N: no mask at all
    (1, 4096, 8, 8, 128, 1023, 0),   # long causal window
]


@pytest.mark.parametrize("B,N,H_q,H_kv,d,left,right", SHAPES)
def test_window_forward(sqa, B, N, H_q, H_kv, d, left, right):
    x = attention_inputs(B, N, H_q, H_kv, d, seed=900 + N + left, device="cuda")
    o, lse = _fwd(sqa, x, left, right)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    ro, rl = attention_forward(f64(x["q"]), f64(x["k"]), f64(x["v"]), False, 1 / math.sqrt(d),
                               window=(left, right))
    assert_close(f64(o), ro, "O")
    assert_close(f64(lse), rl, "LSE")


@pytest.mark.parametrize("B,N,H_q,H_kv,d,left,right", SHAPES)
def test_window_backward(sqa, B, N, H_q, H_kv, d, left, right):
    x = attention_inputs(B, N, H_q, H_kv, d, seed=950 + N + right, with_dout=True, device="cuda")
    o, lse = _fwd(sqa, x, left, right)
    dq, dk, dv = _bwd(sqa, x, o, lse, left, right)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    rq, rk, rv = attention_backward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["do"]), False, 1 / math.sqrt(d),
                                    window=(left, right))
    assert_close(f64(dq), rq, "dQ")
    assert_close(f64(dk), rk, "dK")
    assert_close(f64(dv), rv, "dV")


def test_window_n_zero_is_the_causal_path(sqa):
    """(N, 0) is the causal mask: the same kernel parameters, so the same bits
    as the causal entry point, forward and backward."""
    B, N, H_q, H_kv, d = 2, 600, 8, 4, 64
    x = attention_inputs(B, N, H_q, H_kv, d, seed=31, with_dout=True, device="cuda")
    o, lse = _fwd(sqa, x, N + 5, 0)
    o2, lse2 = run_fwd(sqa, x["q"], x["k"], x["v"], True)
    dq, dk, dv = _bwd(sqa, x, o, lse, N + 5, 0)
    from parity import run_bwd
    dq2, dk2, dv2 = run_bwd(sqa, x["q"], x["k"], x["v"], o2, x["do"], lse2, True)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    assert torch.equal(dq, dq2) and torch.equal(dk, dk2) and torch.equal(dv, dv2)


@pytest.mark.parametrize("left,right", [(4095, 0), (2048, 2048)])
def test_window_full_size_sampled_rows(sqa, left, right):
    """The bench's sliding-window workload (B=1, N=131072, SQA (8,4), d=128):
    128 sampled query rows of every head against the oracle."""
    from sqa_inputs import sample_rows
    B, N, H_q, H_kv, d = 1, 131072, 8, 4, 128
    x = attention_inputs(B, N, H_q, H_kv, d, seed=3, device="cuda")
    o, lse = _fwd(sqa, x, left, right)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    rows = sample_rows(N, 128, seed=left + right)
    ro, rl = attention_forward(f64(x["q"]), f64(x["k"]), f64(x["v"]), False, 1 / math.sqrt(d), rows=rows,
                               window=(left, right))
    assert_close(f64(o[:, rows]), ro, "O rows")
    assert_close(f64(lse[:, :, rows]), rl, "LSE rows")


def test_window_backward_full_size_identities(sqa):
    """The SQA training step of the bench's causal window (N=131072, window
    4096, d=128), checked by identities that hold at any size: every softmax
    row sums to one, so sum_u dV[u, j] = sum over tokens and the group's
    heads of dO, and sum_u dS[t, u] = 0, so sum_u dK[u, j] = 0.  The kernel
    rounds P and dS to bf16 (2^-9 ~ 2e-3 relative per element).  P's rounding
    barely moves the dV identity (measured 5e-5 relative); dS rounding leaves
    sum_u dK at about one bf16 unit of the root-sum-square of the dK rows
    (measured 2.4e-3).  Bounds: 1e-3 and 1e-2."""
    B, N, H_q, H_kv, d, left = 1, 131072, 8, 4, 128, 4095
    x = attention_inputs(B, N, H_q, H_kv, d, seed=3, with_dout=True, device="cuda")
    o, lse = _fwd(sqa, x, left, 0)
    dq, dk, dv = _bwd(sqa, x, o, lse, left, 0)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    G = H_q // H_kv
    do_group = x["do"].double().reshape(B, N, H_kv, G, d).sum(dim=(1, 3))  # [B, H_kv, d]
    sv = dv.double().sum(dim=1)
    rel_v = float((sv - do_group).norm() / do_group.norm())
    sk = dk.double().sum(dim=1)
    rel_k = float(sk.norm() / dk.double().norm(dim=-1).pow(2).sum().sqrt())
    assert rel_v <= 1e-3, rel_v
    assert rel_k <= 1e-2, rel_k
