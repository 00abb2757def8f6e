"""GPU parity of the projection GEMM in every operand layout and of a full SQA
layer training step (forward + backward through the C ABI) against the fp64
oracle.  The layer is the small decoder layer: B=16, N=1024, d_model=256,
d_head=16, causal, weights ~ N(0, 0.02), seed 1; the upstream gradient dY is
~ N(0, 1), seed 11."""

import math

import numpy as np
import pytest
import torch

from oracle import projection, sqa_layer_backward
from parity import assert_close, assert_close_scaled, f64
from sqa_inputs import layer_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sqa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_query_attention_b200 as lib
    return lib


def _bf16(shape, gen, std=1.0):
    return (torch.randn(shape, generator=gen, device="cuda") * std).to(torch.bfloat16)


@pytest.mark.parametrize("a_mn,b_mn,M,N,K", [
    (False, False, 1000, 272, 320),
    (False, True, 16384, 256, 128),   # dX = dY W
    (False, True, 300, 64, 16),
    (True, True, 256, 256, 16384),    # dW = dY^T X
    (True, True, 16, 256, 4096),      # narrow weight (H_kv * d_head = 16)
    (True, False, 128, 128, 256),
    (False, True, 20000, 512, 256),   # 314 tiles: several per persistent CTA, ragged last row tile
    (True, True, 2048, 2048, 512),    # 256 tiles, both operands MN-contiguous
])
def test_gemm_layouts(sqa, a_mn, b_mn, M, N, K):
    g = torch.Generator(device="cuda")
    g.manual_seed(M + 3 * N + 7 * K)
    a = _bf16((K, M) if a_mn else (M, K), g)
    b = _bf16((K, N) if b_mn else (N, K), g, 0.05)
    c = torch.empty((M, N), dtype=torch.float32, device="cuda")
    la = sqa.SQA_MN_CONTIGUOUS if a_mn else sqa.SQA_K_CONTIGUOUS
    lb = sqa.SQA_MN_CONTIGUOUS if b_mn else sqa.SQA_K_CONTIGUOUS
    sqa.sqa_gemm(a, la, b, lb, None, c, sqa.SQA_DT_F32, False, M, N, K)
    sqa.sqa_device_status()
    A = f64(a).T if a_mn else f64(a)   # [M, K]
    Bm = f64(b).T if b_mn else f64(b)  # [N, K]
    assert_close(f64(c), projection(A, Bm), "C")


@pytest.mark.parametrize("M,N,K", [(512, 256, 64), (40000, 256, 64)])
def test_gemm_accumulate(sqa, M, N, K):
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    a, b = _bf16((M, K), g), _bf16((K, N), g, 0.05)
    c0 = torch.randn((M, N), generator=g, device="cuda")
    c = c0.clone()
    sqa.sqa_gemm(a, sqa.SQA_K_CONTIGUOUS, b, sqa.SQA_MN_CONTIGUOUS, None, c, sqa.SQA_DT_F32, True, M, N, K)
    sqa.sqa_device_status()
    assert_close(f64(c), f64(c0) + f64(a) @ f64(b), "C + A B")


@pytest.mark.parametrize("a_mn,b_mn,M,N,K,out,with_bias,acc", [
    (True, True, 256, 256, 16384, "f32", False, False),   # d[Wq; Wk; Wv] = dQKV^T X at the layer's shape
    (True, True, 256, 128, 16384, "f32", False, True),    # dWo = dY^T O, accumulated into C
    (False, False, 384, 48, 8208, "bf16", True, False),   # K-contiguous; ragged N (64-wide tile) and K
    (False, True, 200, 16, 4112, "f32", True, False),     # ragged M, N = 16 in a 64-wide tile
    (True, False, 128, 32, 2048, "bf16", False, False),   # 32-wide tile (K-contiguous B, N <= 32)
    (True, True, 768, 256, 16384, "f32", False, False),   # 24 tiles: clusters smaller than eight
])
def test_gemm_split_k(sqa, a_mn, b_mn, M, N, K, out, with_bias, acc):
    """Products with few output tiles and a long K, which split K over a
    cluster and sum the partial tiles through distributed shared memory:
    parity with the oracle (bias, accumulate, bf16 output), and the same bits
    on a second run (the partials are summed in a fixed order)."""
    g = torch.Generator(device="cuda")
    g.manual_seed(M + 5 * N + 3 * K)
    a = _bf16((K, M) if a_mn else (M, K), g)
    b = _bf16((K, N) if b_mn else (N, K), g, 0.02)
    bias = torch.randn((N,), generator=g, device="cuda") if with_bias else None
    c0 = torch.randn((M, N), generator=g, device="cuda")
    la = sqa.SQA_MN_CONTIGUOUS if a_mn else sqa.SQA_K_CONTIGUOUS
    lb = sqa.SQA_MN_CONTIGUOUS if b_mn else sqa.SQA_K_CONTIGUOUS
    dt, tdt = (sqa.SQA_DT_BF16, torch.bfloat16) if out == "bf16" else (sqa.SQA_DT_F32, torch.float32)
    runs = []
    for _ in range(2):
        c = c0.clone() if acc else torch.empty((M, N), dtype=tdt, device="cuda")
        sqa.sqa_gemm(a, la, b, lb, bias, c, dt, acc, M, N, K)
        runs.append(c)
    sqa.sqa_device_status()
    A = f64(a).T if a_mn else f64(a)
    Bm = f64(b).T if b_mn else f64(b)
    want = projection(A, Bm, None if bias is None else f64(bias))
    if acc:
        want = want + f64(c0)
    assert_close(f64(runs[0]), want, "C")
    assert torch.equal(runs[0], runs[1]), "split-K result differs between two runs"


VARIANTS = {"GQA": (16, 4), "SQA": (8, 4), "sSQA": (8, 8), "xSQA": (4, 4), "xSMQA": (4, 1)}


def layer_train_step(sqa, x, dy, B, N, H_q, H_kv, dh, dm):
    """Forward and backward of the layer with the library's kernels only.
    Returns y and the gradients (dx, dwq, dwk, dwv, dwo) as device tensors."""
    M = B * N
    K_, L, Q = sqa.SQA_K_CONTIGUOUS, sqa.SQA_MN_CONTIGUOUS, sqa.SQA_DT_BF16
    F32 = sqa.SQA_DT_F32
    dev = dy.device
    bf = torch.bfloat16
    q = torch.empty((M, H_q * dh), dtype=bf, device=dev)
    k = torch.empty((M, H_kv * dh), dtype=bf, device=dev)
    v = torch.empty((M, H_kv * dh), dtype=bf, device=dev)
    o = torch.empty((M, H_q * dh), dtype=bf, device=dev)
    lse = torch.empty((B, H_q, N), dtype=torch.float32, device=dev)
    y = torch.empty((M, dm), dtype=torch.float32, device=dev)
    sqa.sqa_proj(x["x"], x["wq"], None, q, Q, M, dm, H_q * dh)
    sqa.sqa_proj(x["x"], x["wk"], None, k, Q, M, dm, H_kv * dh)
    sqa.sqa_proj(x["x"], x["wv"], None, v, Q, M, dm, H_kv * dh)
    sqa.sqa_attn_fwd_ex(q, k, v, o, Q, lse, B, N, H_q, H_kv, dh, True, 1 / math.sqrt(dh))
    sqa.sqa_proj(o, x["wo"], None, y, F32, M, H_q * dh, dm)
    # backward
    do = torch.empty_like(o)
    dwo = torch.empty((dm, H_q * dh), dtype=torch.float32, device=dev)
    sqa.sqa_gemm(dy, K_, x["wo"], L, None, do, Q, False, M, H_q * dh, dm)        # dO = dY Wo
    sqa.sqa_gemm(dy, L, o, L, None, dwo, F32, False, dm, H_q * dh, M)            # dWo = dY^T O
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    wsb = sqa.sqa_attn_bwd_workspace_size(B, N, H_q, H_kv, dh)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    sqa.sqa_attn_bwd(q, k, v, o, Q, do, lse, dq, dk, dv, Q, B, N, H_q, H_kv, dh, True, 1 / math.sqrt(dh), ws, wsb)
    dx = torch.empty((M, dm), dtype=torch.float32, device=dev)
    grads = {"dx": dx}
    for i, (name, g_, width) in enumerate((("wq", dq, H_q), ("wk", dk, H_kv), ("wv", dv, H_kv))):
        dw = torch.empty((width * dh, dm), dtype=torch.float32, device=dev)
        sqa.sqa_gemm(g_, L, x["x"], L, None, dw, F32, False, width * dh, dm, M)     # dW = dG^T X
        sqa.sqa_gemm(g_, K_, x[name], L, None, dx, F32, i > 0, M, dm, width * dh)  # dX += dG W
        grads["d" + name] = dw
    grads["dwo"] = dwo
    return y, grads


@pytest.mark.parametrize("name", list(VARIANTS))
def test_layer_training_step(sqa, name):
    H_q, H_kv = VARIANTS[name]
    B, N, dm, dh = 16, 1024, 256, 16
    x = layer_inputs(B, N, dm, H_q, H_kv, dh, seed=1, device="cuda")
    gen = torch.Generator(device="cuda")
    gen.manual_seed(11)
    dy = torch.randn((B * N, dm), generator=gen, device="cuda").to(torch.bfloat16)
    y, grads = layer_train_step(sqa, x, dy, B, N, H_q, H_kv, dh, dm)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    ref = sqa_layer_backward(f64(x["x"]), f64(x["wq"]), f64(x["wk"]), f64(x["wv"]), f64(x["wo"]), f64(dy),
                             B, N, H_q, H_kv, dh, causal=True)
    for key in ("dx", "dwq", "dwk", "dwv", "dwo"):
        got = f64(grads[key])
        assert np.isfinite(got).all()
        assert_close_scaled(got, ref[key], key)


def layer_train_step_fused(sqa, x, dy, B, N, H_q, H_kv, dh, dm):
    """The same layer with the input projection fused: one GEMM with the
    concatenated weight [Wq; Wk; Wv] writes a packed QKV buffer, the attention
    reads and its backward writes the packed layout, and the input
    projection's backward is one GEMM for dX and one for d[Wq; Wk; Wv]
    (10 launches per training step instead of 15)."""
    M = B * N
    KC, MN, BF, F32 = sqa.SQA_K_CONTIGUOUS, sqa.SQA_MN_CONTIGUOUS, sqa.SQA_DT_BF16, sqa.SQA_DT_F32
    dev = dy.device
    W = (H_q + 2 * H_kv) * dh
    w_qkv = torch.cat([x["wq"], x["wk"], x["wv"]], dim=0).contiguous()
    qkv = torch.empty((M, W), dtype=torch.bfloat16, device=dev)
    o = torch.empty((M, H_q * dh), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H_q, N), dtype=torch.float32, device=dev)
    y = torch.empty((M, dm), dtype=torch.float32, device=dev)
    sc = 1 / math.sqrt(dh)
    sqa.sqa_proj(x["x"], w_qkv, None, qkv, BF, M, dm, W)
    sqa.sqa_attn_fwd_packed(qkv, o, BF, lse, B, N, H_q, H_kv, dh, True, sc)
    sqa.sqa_proj(o, x["wo"], None, y, F32, M, H_q * dh, dm)
    do = torch.empty_like(o)
    dwo = torch.empty((dm, H_q * dh), dtype=torch.float32, device=dev)
    sqa.sqa_gemm(dy, KC, x["wo"], MN, None, do, BF, False, M, H_q * dh, dm)
    sqa.sqa_gemm(dy, MN, o, MN, None, dwo, F32, False, dm, H_q * dh, M)
    dqkv = torch.empty_like(qkv)
    wsb = sqa.sqa_attn_bwd_workspace_size(B, N, H_q, H_kv, dh)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    sqa.sqa_attn_bwd_packed(qkv, o, BF, do, lse, dqkv, BF, B, N, H_q, H_kv, dh, True, sc, ws, wsb)
    dx = torch.empty((M, dm), dtype=torch.float32, device=dev)
    dw = torch.empty((W, dm), dtype=torch.float32, device=dev)
    sqa.sqa_gemm(dqkv, KC, w_qkv, MN, None, dx, F32, False, M, dm, W)   # dX = dQKV [Wq; Wk; Wv]
    sqa.sqa_gemm(dqkv, MN, x["x"], MN, None, dw, F32, False, W, dm, M)  # d[Wq; Wk; Wv] = dQKV^T X
    a, b = H_q * dh, (H_q + H_kv) * dh
    return y, {"dx": dx, "dwq": dw[:a], "dwk": dw[a:b], "dwv": dw[b:], "dwo": dwo}


@pytest.mark.parametrize("name", list(VARIANTS))
def test_layer_training_step_fused_qkv(sqa, name):
    H_q, H_kv = VARIANTS[name]
    B, N, dm, dh = 16, 1024, 256, 16
    x = layer_inputs(B, N, dm, H_q, H_kv, dh, seed=1, device="cuda")
    gen = torch.Generator(device="cuda")
    gen.manual_seed(11)
    dy = torch.randn((B * N, dm), generator=gen, device="cuda").to(torch.bfloat16)
    y, grads = layer_train_step_fused(sqa, x, dy, B, N, H_q, H_kv, dh, dm)
    y2, grads2 = layer_train_step(sqa, x, dy, B, N, H_q, H_kv, dh, dm)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    ref = sqa_layer_backward(f64(x["x"]), f64(x["wq"]), f64(x["wk"]), f64(x["wv"]), f64(x["wo"]), f64(dy),
                             B, N, H_q, H_kv, dh, causal=True)
    for key in ("dx", "dwq", "dwk", "dwv", "dwo"):
        assert_close_scaled(f64(grads[key]), ref[key], key)
    # The attention output, and so y and dWo, are the same bits on both paths.
    assert torch.equal(y, y2)
    assert torch.equal(grads["dwo"], grads2["dwo"])
