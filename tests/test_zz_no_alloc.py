"""sqa_attn_bwd_static: the backward for callers that cannot allocate device
memory (plugins handed only input/output pointers by a framework that owns
the GPU's memory, services that forbid allocation while running).  It uses
the library's fixed device scratch array instead of a caller workspace.

Checked through the C ABI against sqa_attn_bwd (the entry point that takes a
workspace) on two calls in a row with different shapes, so the second call
runs on scratch that still holds the first call's contents.  Both entry
points run the same deterministic kernels on the same inputs, so their
gradients must be the same bits: a stale scratch value read by the second
call would show even if it stayed within the parity tolerance.  This file is
collected last on purpose.
"""

import math

import pytest
import torch

from parity import run_bwd, run_fwd
from sqa_inputs import attention_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sqa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_query_attention_b200 as lib
    return lib


def _static_bwd(sqa, x, o, lse, causal):
    B, N, H_q, d = x["q"].shape
    H_kv = x["k"].shape[2]
    # Outputs start as NaN so a partial write would show.
    dq = torch.full((B, N, H_q, d), float("nan"), dtype=torch.float32, device="cuda")
    dk = torch.full((B, N, H_kv, d), float("nan"), dtype=torch.float32, device="cuda")
    dv = torch.full((B, N, H_kv, d), float("nan"), dtype=torch.float32, device="cuda")
    od = sqa.SQA_DT_BF16 if o.dtype == torch.bfloat16 else sqa.SQA_DT_F32
    sqa.sqa_attn_bwd_static(x["q"], x["k"], x["v"], o, od, x["do"], lse, dq, dk, dv, sqa.SQA_DT_F32,
                            B, N, H_q, H_kv, d, causal, 1 / math.sqrt(d))
    return dq, dk, dv


def test_static_scratch_backward_matches_workspace_backward(sqa):
    shapes = [
        (2, 1000, 8, 4, 64, True, 101),   # ragged N, SQA head counts
        (1, 384, 4, 1, 128, False, 102),  # smaller problem on stale scratch
    ]
    for B, N, H_q, H_kv, d, causal, seed in shapes:
        x = attention_inputs(B, N, H_q, H_kv, d, seed, with_dout=True, device="cuda")
        o, lse = run_fwd(sqa, x["q"], x["k"], x["v"], causal)
        want = run_bwd(sqa, x["q"], x["k"], x["v"], o, x["do"], lse, causal)
        got = _static_bwd(sqa, x, o, lse, causal)
        torch.cuda.synchronize()
        sqa.sqa_device_status()
        for name, g, w in zip(("dQ", "dK", "dV"), got, want):
            assert torch.isfinite(g).all(), f"{name}: unwritten (NaN) entries"
            assert torch.equal(g, w), f"{name} B={B} N={N} H_q={H_q} H_kv={H_kv} d={d}: not bitwise equal"


def test_static_scratch_rejects_oversized_problem(sqa):
    B, N, H_q, H_kv, d = 1, 262144, 16, 16, 16
    need = sqa.sqa_attn_bwd_workspace_size(B, N, H_q, H_kv, d)
    assert need > 16 << 20
    # Real buffers of the stated size, so nothing could run out of bounds.
    q = torch.zeros((B, N, H_q, d), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((B, N, H_kv, d), dtype=torch.bfloat16, device="cuda")
    o = torch.zeros((B, N, H_q, d), dtype=torch.float32, device="cuda")
    lse = torch.zeros((B, H_q, N), dtype=torch.float32, device="cuda")
    g = torch.zeros((B, N, H_q, d), dtype=torch.float32, device="cuda")
    status = sqa.library().sqa_attn_bwd_static(
        q.data_ptr(), kv.data_ptr(), kv.data_ptr(), o.data_ptr(), sqa.SQA_DT_F32, q.data_ptr(), lse.data_ptr(),
        g.data_ptr(), g.data_ptr(), g.data_ptr(), sqa.SQA_DT_F32, B, N, H_q, H_kv, d, 1, 0.25,
        torch.cuda.current_stream().cuda_stream)
    assert status == sqa.SQA_ERR_UNSUPPORTED
