"""Chains of launches with no synchronisation between them.

Every kernel is launched as a programmatic dependent of the previous one on
the stream: it may start its set-up while that kernel finishes and must wait
for it before touching global memory.  These tests run chains in which each
launch reads what the previous one wrote (read after write) and overwrites
what the previous one still reads (write after read), with buffers and
workspaces reused from step to step, and compare every result bit for bit
with the same computation run one call at a time with a synchronise after
each.  No kernel uses atomics, so equal inputs must give equal bits."""

import math

import pytest
import torch

from sqa_inputs import attention_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sqa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_query_attention_b200 as lib
    return lib


def _fwd(sqa, x, out, causal):
    B, N, H_q, d = x["q"].shape
    sqa.sqa_attn_fwd_ex(x["q"], x["k"], x["v"], out, sqa.SQA_DT_BF16, None, B, N, H_q, x["k"].shape[2], d, causal,
                        1 / math.sqrt(d))


@pytest.mark.parametrize("d,causal,B,N,H_q,H_kv", [(64, True, 2, 640, 8, 4), (128, False, 2, 640, 8, 4),
                                                   (16, True, 2, 640, 8, 4), (128, False, 1, 40883, 4, 4)])
def test_forward_then_projection_chain(sqa, d, causal, B, N, H_q, H_kv):
    """fwd(X_s) -> O, then Y_s = O W^T, for three inputs through ONE O
    buffer: each projection reads the O just written, and the next forward
    overwrites O right after that projection was launched.  The last shape
    runs the forward as two launches (two-tile kernel, then the split kernel
    on the remaining query tiles, which waits for the first only before it
    exits)."""
    Nout = 96
    xs = [attention_inputs(B, N, H_q, H_kv, d, seed=900 + s, device="cuda") for s in range(3)]
    g = torch.Generator(device="cuda")
    g.manual_seed(901)
    w = (0.05 * torch.randn((Nout, H_q * d), generator=g, device="cuda")).to(torch.bfloat16)
    M, K = B * N, H_q * d

    want = []
    for x in xs:
        o = torch.empty((B, N, H_q, d), dtype=torch.bfloat16, device="cuda")
        _fwd(sqa, x, o, causal)
        torch.cuda.synchronize()
        y = torch.empty((M, Nout), dtype=torch.float32, device="cuda")
        sqa.sqa_proj(o, w, None, y, sqa.SQA_DT_F32, M, K, Nout)
        torch.cuda.synchronize()
        want.append(y)

    o = torch.empty((B, N, H_q, d), dtype=torch.bfloat16, device="cuda")
    got = [torch.empty((M, Nout), dtype=torch.float32, device="cuda") for _ in xs]
    for x, y in zip(xs, got):
        _fwd(sqa, x, o, causal)
        sqa.sqa_proj(o, w, None, y, sqa.SQA_DT_F32, M, K, Nout)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    for s, (a, b) in enumerate(zip(got, want)):
        assert torch.equal(a, b), f"chain step {s} differs from the synchronised run"


def test_decode_steps_share_one_workspace(sqa):
    """Four decode steps (multi-chunk plan, so each is decode + combine)
    through one workspace: step s+1's decode overwrites the partial results
    that step s's combine reads."""
    B, n_new, H_q, H_kv, d, L_max = 4, 1, 8, 4, 128, 6000
    lens = torch.tensor([6000, 5000, 1234, 4097], dtype=torch.int32, device="cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(902)
    kc = torch.randn((B, L_max, H_kv, d), generator=g, device="cuda").to(torch.bfloat16)
    vc = torch.randn((B, L_max, H_kv, d), generator=g, device="cuda").to(torch.bfloat16)
    qs = [torch.randn((B, n_new, H_q, d), generator=g, device="cuda").to(torch.bfloat16) for _ in range(4)]
    wsb = sqa.sqa_attn_decode_workspace_size(B, n_new, H_q, H_kv, d, L_max)
    assert wsb > 0
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")

    def step(q, out):
        sqa.sqa_attn_decode(q, kc, vc, lens, out, sqa.SQA_DT_F32, None, B, n_new, H_q, H_kv, d, L_max,
                            1 / math.sqrt(d), ws, wsb)

    want = []
    for q in qs:
        out = torch.empty((B, n_new, H_q, d), dtype=torch.float32, device="cuda")
        step(q, out)
        torch.cuda.synchronize()
        want.append(out)
    got = [torch.empty((B, n_new, H_q, d), dtype=torch.float32, device="cuda") for _ in qs]
    for q, out in zip(qs, got):
        step(q, out)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    for s, (a, b) in enumerate(zip(got, want)):
        assert torch.equal(a, b), f"decode step {s} differs from the synchronised run"


def test_training_chain_reuses_every_buffer(sqa):
    """Two training steps of the attention core (forward, backward =
    preprocess + dK/dV + dQ, then a GEMM that reads dQ) through the same O,
    LSE, gradient and workspace buffers, with no synchronisation."""
    B, N, H_q, H_kv, d = 2, 1024, 8, 4, 64
    xs = [attention_inputs(B, N, H_q, H_kv, d, seed=910 + s, with_dout=True, device="cuda") for s in range(2)]
    scale = 1 / math.sqrt(d)
    M, K, Nout = B * N, H_q * d, 64
    g = torch.Generator(device="cuda")
    g.manual_seed(903)
    w = (0.05 * torch.randn((Nout, K), generator=g, device="cuda")).to(torch.bfloat16)
    wsb = sqa.sqa_attn_bwd_workspace_size(B, N, H_q, H_kv, d)

    def bufs():
        return {"o": torch.empty((B, N, H_q, d), dtype=torch.bfloat16, device="cuda"),
                "lse": torch.empty((B, H_q, N), dtype=torch.float32, device="cuda"),
                "dq": torch.empty((B, N, H_q, d), dtype=torch.bfloat16, device="cuda"),
                "dk": torch.empty((B, N, H_kv, d), dtype=torch.bfloat16, device="cuda"),
                "dv": torch.empty((B, N, H_kv, d), dtype=torch.bfloat16, device="cuda"),
                "ws": torch.empty(wsb, dtype=torch.uint8, device="cuda")}

    def train_step(x, b, y, sync):
        sqa.sqa_attn_fwd_ex(x["q"], x["k"], x["v"], b["o"], sqa.SQA_DT_BF16, b["lse"], B, N, H_q, H_kv, d, True,
                            scale)
        if sync:
            torch.cuda.synchronize()
        sqa.sqa_attn_bwd(x["q"], x["k"], x["v"], b["o"], sqa.SQA_DT_BF16, x["do"], b["lse"], b["dq"], b["dk"],
                         b["dv"], sqa.SQA_DT_BF16, B, N, H_q, H_kv, d, True, scale, b["ws"], wsb)
        if sync:
            torch.cuda.synchronize()
        sqa.sqa_proj(b["dq"], w, None, y, sqa.SQA_DT_F32, M, K, Nout)
        if sync:
            torch.cuda.synchronize()
        return [y] + [b[n] for n in ("dk", "dv")]

    want = []
    for x in xs:
        y = torch.empty((M, Nout), dtype=torch.float32, device="cuda")
        want.append([t.clone() for t in train_step(x, bufs(), y, sync=True)])
    shared = bufs()
    got = []
    for x in xs:
        y = torch.empty((M, Nout), dtype=torch.float32, device="cuda")
        res = train_step(x, shared, y, sync=False)
        # dK and dV of this step are copied out on the stream, before the next
        # step's backward overwrites them.
        got.append([res[0]] + [t.clone() for t in res[1:]])
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    for s, (gs, ws_) in enumerate(zip(got, want)):
        for name, a, b in zip(("Y = dQ W^T", "dK", "dV"), gs, ws_):
            assert torch.equal(a, b), f"step {s}: {name} differs from the synchronised run"
