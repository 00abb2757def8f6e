"""GPU parity of cross / memory attention (N_q query tokens, N_kv key/value
tokens of another sequence, no mask) against the fp64 oracle: forward output
and log-sum-exp, and all three gradients."""

import math

import pytest
import torch

from oracle import attention_backward, attention_forward
from parity import assert_close, f64
from sqa_inputs import cross_attention_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sqa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_query_attention_b200 as lib
    return lib


def _fwd(sqa, x, out_dtype=torch.float32):
    B, N_q, H_q, d = x["q"].shape
    N_kv, H_kv = x["k"].shape[1], x["k"].shape[2]
    out = torch.empty((B, N_q, H_q, d), dtype=out_dtype, device="cuda")
    lse = torch.empty((B, H_q, N_q), dtype=torch.float32, device="cuda")
    dt = sqa.SQA_DT_BF16 if out_dtype == torch.bfloat16 else sqa.SQA_DT_F32
    sqa.sqa_attn_fwd_cross(x["q"], x["k"], x["v"], out, dt, lse, B, N_q, N_kv, H_q, H_kv, d, 1 / math.sqrt(d))
    return out, lse


def _bwd(sqa, x, o, lse, grad_dtype=torch.float32):
    B, N_q, H_q, d = x["q"].shape
    N_kv, H_kv = x["k"].shape[1], x["k"].shape[2]
    dq = torch.empty_like(x["q"], dtype=grad_dtype)
    dk = torch.empty_like(x["k"], dtype=grad_dtype)
    dv = torch.empty_like(x["v"], dtype=grad_dtype)
    wsb = sqa.sqa_attn_bwd_workspace_size(B, N_q, H_q, H_kv, d)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    od = sqa.SQA_DT_BF16 if o.dtype == torch.bfloat16 else sqa.SQA_DT_F32
    gd = sqa.SQA_DT_BF16 if grad_dtype == torch.bfloat16 else sqa.SQA_DT_F32
    sqa.sqa_attn_bwd_cross(x["q"], x["k"], x["v"], o, od, x["do"], lse, dq, dk, dv, gd, B, N_q, N_kv, H_q, H_kv,
                           d, 1 / math.sqrt(d), ws, wsb)
    return dq, dk, dv


# Memory reads from a short state (N_kv < N_q), an encoder of a different
# length (N_kv > N_q), single tokens on either side, and lengths that are and
# are not multiples of the 128-key tile.
SHAPES = [
    (2, 300, 1000, 8, 4, 64),
    (1, 1000, 77, 8, 2, 128),
    (1, 1, 513, 4, 4, 64),
    (2, 257, 1, 4, 1, 32),
    (1, 128, 384, 16, 4, 16),
    (3, 200, 1536, 4, 2, 128),
    (1, 129, 4100, 6, 2, 64),
]


@pytest.mark.parametrize("B,N_q,N_kv,H_q,H_kv,d", SHAPES)
def test_cross_forward(sqa, B, N_q, N_kv, H_q, H_kv, d):
    x = cross_attention_inputs(B, N_q, N_kv, H_q, H_kv, d, seed=N_q * 31 + N_kv, device="cuda")
    o, lse = _fwd(sqa, x)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    ro, rl = attention_forward(f64(x["q"]), f64(x["k"]), f64(x["v"]), False, 1 / math.sqrt(d))
    assert_close(f64(o), ro, "O")
    assert_close(f64(lse), rl, "LSE")


@pytest.mark.parametrize("B,N_q,N_kv,H_q,H_kv,d", SHAPES)
def test_cross_backward(sqa, B, N_q, N_kv, H_q, H_kv, d):
    x = cross_attention_inputs(B, N_q, N_kv, H_q, H_kv, d, seed=N_q * 37 + N_kv, with_dout=True, device="cuda")
    o, lse = _fwd(sqa, x)
    dq, dk, dv = _bwd(sqa, x, o, lse)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    rq, rk, rv = attention_backward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["do"]), False, 1 / math.sqrt(d))
    assert_close(f64(dq), rq, "dQ")
    assert_close(f64(dk), rk, "dK")
    assert_close(f64(dv), rv, "dV")


def test_cross_bf16_outputs(sqa):
    x = cross_attention_inputs(2, 640, 200, 8, 4, 64, seed=91, with_dout=True, device="cuda")
    o, lse = _fwd(sqa, x, out_dtype=torch.bfloat16)
    dq, dk, dv = _bwd(sqa, x, o, lse, grad_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    scale = 1 / math.sqrt(64)
    ro, _ = attention_forward(f64(x["q"]), f64(x["k"]), f64(x["v"]), False, scale)
    rq, rk, rv = attention_backward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["do"]), False, scale)
    assert_close(f64(o), ro, "O")
    assert_close(f64(dq), rq, "dQ")
    assert_close(f64(dk), rk, "dK")
    assert_close(f64(dv), rv, "dV")


def test_cross_equal_lengths_match_self_attention(sqa):
    """N_q = N_kv without a mask is the non-causal self-attention call: the
    same kernels on the same bits give the same bits."""
    x = cross_attention_inputs(1, 700, 700, 8, 4, 64, seed=5, device="cuda")
    o, lse = _fwd(sqa, x)
    o2 = torch.empty_like(o)
    lse2 = torch.empty_like(lse)
    sqa.sqa_attn_fwd_ex(x["q"], x["k"], x["v"], o2, sqa.SQA_DT_F32, lse2, 1, 700, 8, 4, 64, False,
                        1 / math.sqrt(64))
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)


# Few key tiles against many queries: each key tile's dK/dV steps are split
# over a cluster of 2, 4 or 8 CTAs and the partial dK/dV summed through
# distributed shared memory.  Ragged key lengths, G = 3 (the CTAs' shares of
# the steps end inside a head), d from 16 to 128, non-causal self-attention
# (N_q = N_kv), and the same bits on a second run (fixed summation order).
SPLIT_SHAPES = [
    (1, 4096, 1024, 8, 4, 128),   # 32 key tiles x heads: clusters of 4
    (1, 1000, 300, 6, 2, 64),     # G = 3, shares cross head boundaries
    (2, 2048, 77, 4, 4, 32),      # one ragged key tile per head
    (1, 3000, 200, 4, 1, 16),     # clusters of 8
    (1, 2048, 2048, 8, 4, 64),    # non-causal self-attention: clusters of 2
]


# Few query tiles against many keys: each query tile's key sub-tiles are
# split over a cluster in the dQ kernel and the partial dQ rows summed.
DQ_SPLIT_SHAPES = [
    (1, 300, 5000, 8, 4, 128),    # ragged N_q and N_kv
    (2, 129, 2048, 4, 4, 64),     # a query tile with one token
    (1, 64, 1000, 6, 2, 32),      # G = 3, clusters of 2
    (1, 100, 3000, 4, 1, 16),     # four heads per tile (g = 4)
]


@pytest.mark.parametrize("B,N_q,N_kv,H_q,H_kv,d", SPLIT_SHAPES + DQ_SPLIT_SHAPES)
def test_cross_backward_split_key_tiles(sqa, B, N_q, N_kv, H_q, H_kv, d):
    x = cross_attention_inputs(B, N_q, N_kv, H_q, H_kv, d, seed=N_q * 41 + N_kv, with_dout=True, device="cuda")
    o, lse = _fwd(sqa, x)
    g1 = _bwd(sqa, x, o, lse)
    g2 = _bwd(sqa, x, o, lse)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    rq, rk, rv = attention_backward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["do"]), False, 1 / math.sqrt(d))
    assert_close(f64(g1[0]), rq, "dQ")
    assert_close(f64(g1[1]), rk, "dK")
    assert_close(f64(g1[2]), rv, "dV")
    for a, b in zip(g1, g2):
        assert torch.equal(a, b), "gradients differ between two runs"


# Few query tiles against many keys (d = 128, unmasked): every token block's
# key range is split over a cluster of 2, 4 or 8 CTAs and the rows' partial
# O, running max and sum merged through distributed shared memory.  Ragged
# N_q (a block whose second tile is partly or wholly past N) and N_kv, G = 3
# (one head per tile row group), fp32 and bf16 outputs with the LSE, and the
# same bits on a second run.
FWD_SPLIT_SHAPES = [
    (1, 300, 5000, 8, 4, torch.float32),    # clusters of 8
    (2, 129, 2048, 4, 4, torch.bfloat16),   # clusters of 4, one token in the second tile
    (1, 64, 1000, 6, 2, torch.float32),     # G = 3, clusters of 2
    (1, 1024, 1024, 8, 4, torch.bfloat16),  # non-causal self-attention shape
]


@pytest.mark.parametrize("B,N_q,N_kv,H_q,H_kv,odt", FWD_SPLIT_SHAPES)
def test_cross_forward_split_key_range(sqa, B, N_q, N_kv, H_q, H_kv, odt):
    d = 128
    x = cross_attention_inputs(B, N_q, N_kv, H_q, H_kv, d, seed=N_q * 43 + N_kv, device="cuda")
    o1, l1 = _fwd(sqa, x, out_dtype=odt)
    o2, l2 = _fwd(sqa, x, out_dtype=odt)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    ro, rl = attention_forward(f64(x["q"]), f64(x["k"]), f64(x["v"]), False, 1 / math.sqrt(d))
    assert_close(f64(o1), ro, "O")
    assert_close(f64(l1), rl, "LSE")
    assert torch.equal(o1, o2) and torch.equal(l1, l2), "forward differs between two runs"
    # Without the LSE output the merged O is the same.
    o3 = torch.empty_like(o1)
    dt = sqa.SQA_DT_BF16 if odt == torch.bfloat16 else sqa.SQA_DT_F32
    sqa.sqa_attn_fwd_cross(x["q"], x["k"], x["v"], o3, dt, None, B, N_q, N_kv, H_q, H_kv, d, 1 / math.sqrt(d))
    torch.cuda.synchronize()
    assert torch.equal(o1, o3), "O differs without the LSE output"
