"""GPU parity of the reduced-width projections and of the small SQA decoder
layer (projections + causal core + output projection) against the oracle."""

import math

import numpy as np
import pytest
import torch

from oracle import projection, sqa_layer_forward
from parity import assert_close, f64, run_fwd
from sqa_inputs import layer_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sqa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_query_attention_b200 as lib
    return lib


def _proj(sqa, x, w, bias=None, out_dtype=torch.float32):
    M, K = x.shape
    Nout = w.shape[0]
    y = torch.empty((M, Nout), dtype=out_dtype, device=x.device)
    dt = sqa.SQA_DT_BF16 if out_dtype == torch.bfloat16 else sqa.SQA_DT_F32
    sqa.sqa_proj(x, w, bias, y, dt, M, K, Nout)
    return y


@pytest.mark.parametrize("M,K,Nout", [
    (16384, 256, 256), (16384, 256, 128), (16384, 256, 64), (16384, 256, 16),
    (16384, 64, 256), (16384, 128, 256),
    (1000, 256, 48), (129, 32, 16), (1, 16, 16), (300, 320, 272), (4096, 2048, 2048),
])
def test_proj_shapes(sqa, M, K, Nout):
    g = torch.Generator(device="cuda")
    g.manual_seed(M + K + Nout)
    x = torch.randn((M, K), generator=g, device="cuda").to(torch.bfloat16)
    w = (torch.randn((Nout, K), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    y = _proj(sqa, x, w)
    sqa.sqa_device_status()
    assert_close(f64(y), projection(f64(x), f64(w)), "Y")


def test_proj_bias_and_bf16(sqa):
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    x = torch.randn((777, 256), generator=g, device="cuda").to(torch.bfloat16)
    w = (torch.randn((128, 256), generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    bias = torch.randn((128,), generator=g, device="cuda")
    y = _proj(sqa, x, w, bias=bias, out_dtype=torch.bfloat16)
    sqa.sqa_device_status()
    assert_close(f64(y), projection(f64(x), f64(w), f64(bias)), "Y")


@pytest.mark.parametrize("M,K,Nout,bf16_out", [(4100, 528, 2320, True), (4100, 528, 2320, False),
                                                (8200, 1008, 784, True)])
def test_proj_pair_tiles(sqa, M, K, Nout, bf16_out):
    """Products large enough to run on CTA pairs (256 x 256 tiles, two SMs per
    tile): ragged M, Nout and K (M not a multiple of 256, Nout of 256, K of
    64), with a bias."""
    g = torch.Generator(device="cuda")
    g.manual_seed(M + 3 * K + Nout)
    x = torch.randn((M, K), generator=g, device="cuda").to(torch.bfloat16)
    w = (torch.randn((Nout, K), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    bias = torch.randn((Nout,), generator=g, device="cuda")
    y = _proj(sqa, x, w, bias=bias, out_dtype=torch.bfloat16 if bf16_out else torch.float32)
    sqa.sqa_device_status()
    assert_close(f64(y), projection(f64(x), f64(w), f64(bias)), "Y")


def test_gemm_pair_tiles_accumulate(sqa):
    """C += A B^T twice into an fp32 C on the pair path (sqa_gemm, both
    operands K-contiguous): the epilogue adds to what C holds."""
    M, K, N = 3000, 256, 1024
    g = torch.Generator(device="cuda")
    g.manual_seed(77)
    a = torch.randn((M, K), generator=g, device="cuda").to(torch.bfloat16)
    b = (torch.randn((N, K), generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    c0 = torch.randn((M, N), generator=g, device="cuda")
    c = c0.clone()
    KC = sqa.SQA_K_CONTIGUOUS
    sqa.sqa_gemm(a, KC, b, KC, None, c, sqa.SQA_DT_F32, True, M, N, K)
    sqa.sqa_gemm(a, KC, b, KC, None, c, sqa.SQA_DT_F32, True, M, N, K)
    sqa.sqa_device_status()
    assert_close(f64(c), f64(c0) + 2 * projection(f64(a), f64(b)), "C")


def test_proj_bench_size_sampled_rows(sqa):
    """The bench's projection, M = 32768, N = K = 4096, bf16 out, on the pair
    path; 256 seeded rows against the oracle."""
    M, K, N = 32768, 4096, 4096
    g = torch.Generator(device="cuda")
    g.manual_seed(6)
    x = torch.randn((M, K), generator=g, device="cuda").to(torch.bfloat16)
    w = (0.02 * torch.randn((N, K), generator=g, device="cuda")).to(torch.bfloat16)
    y = _proj(sqa, x, w, out_dtype=torch.bfloat16)
    sqa.sqa_device_status()
    rows = np.sort(np.random.default_rng(6).choice(M, 256, replace=False))
    ri = torch.as_tensor(rows, device="cuda")
    assert_close(f64(y[ri]), projection(f64(x[ri]), f64(w)), "Y rows")


VARIANTS = {"GQA": (16, 4), "SQA": (8, 4), "sSQA": (8, 8), "xSQA": (4, 4), "xSMQA": (4, 1)}


@pytest.mark.parametrize("name", list(VARIANTS))
def test_small_decoder_layer(sqa, name):
    """B=16, N=1024, d_model=256, d_head=16, causal; x ~ N(0,1), weights ~ N(0, 0.02),
    seed 1.  Q/K/V projections -> causal SQA core -> output projection."""
    H_q, H_kv = VARIANTS[name]
    B, N, dm, dh = 16, 1024, 256, 16
    x = layer_inputs(B, N, dm, H_q, H_kv, dh, seed=1, device="cuda")
    q = _proj(sqa, x["x"], x["wq"], out_dtype=torch.bfloat16).view(B, N, H_q, dh)
    k = _proj(sqa, x["x"], x["wk"], out_dtype=torch.bfloat16).view(B, N, H_kv, dh)
    v = _proj(sqa, x["x"], x["wv"], out_dtype=torch.bfloat16).view(B, N, H_kv, dh)
    o, _ = run_fwd(sqa, q, k, v, True, out_dtype=torch.bfloat16, with_lse=False)
    y = _proj(sqa, o.view(B * N, H_q * dh), x["wo"])
    sqa.sqa_device_status()
    ref = sqa_layer_forward(f64(x["x"]), f64(x["wq"]), f64(x["wk"]), f64(x["wv"]), f64(x["wo"]),
                            B, N, H_q, H_kv, dh, causal=True)
    assert_close(f64(y), ref["y"], "y")
    assert_close(f64(o).reshape(B * N, H_q * dh), ref["o"], "attention output")
    assert np.isfinite(f64(y)).all()
