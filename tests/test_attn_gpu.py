"""GPU parity of the SQA attention core (forward) against the fp64 oracle,
through the C ABI, on seeded inputs."""

import math

import numpy as np
import pytest
import torch

from oracle import attention_forward
from parity import assert_close, f64, run_fwd
from sqa_inputs import attention_inputs, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sqa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_query_attention_b200 as lib
    return lib


def _oracle_fwd(x, causal, scale=None, rows=None):
    d = x["q"].shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    return attention_forward(f64(x["q"]), f64(x["k"]), f64(x["v"]), causal, scale, rows=rows)


def _check_fwd(sqa, B, N, H_q, H_kv, d, causal, seed, out_dtype=torch.float32, scale=None, mult=1.0):
    x = attention_inputs(B, N, H_q, H_kv, d, seed, device="cuda")
    if mult != 1.0:
        x = {n: (t.float() * mult).to(torch.bfloat16) for n, t in x.items()}
    o, lse = run_fwd(sqa, x["q"], x["k"], x["v"], causal, scale=scale, out_dtype=out_dtype)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    o_ref, lse_ref = _oracle_fwd(x, causal, scale)
    assert_close(f64(o), o_ref, "O")
    assert_close(f64(lse), lse_ref, "LSE")


def test_config_small_causal_decoder(sqa):
    """B=2, N=256, H_q=4, H_kv=2, d=32, causal, fp32 output [B,N,H_q*d], seed 0."""
    x = attention_inputs(2, 256, 4, 2, 32, seed=0, device="cuda")
    out = torch.empty((2, 256, 4 * 32), dtype=torch.float32, device="cuda")
    sqa.sqa_attn_fwd(x["q"], x["k"], x["v"], out, 2, 256, 4, 2, 32, True, 1 / math.sqrt(32))
    sqa.sqa_device_status()
    o_ref, _ = _oracle_fwd(x, True)
    assert_close(f64(out), o_ref.reshape(2, 256, 128), "O")


def _sweep():
    cases = []
    Ns = [1, 2, 127, 128, 129, 255, 256, 1000]
    Gs = [1, 2, 4, 8, 16]
    i = 0
    for d in (16, 32, 64, 128):
        for N in Ns:
            G = Gs[i % len(Gs)]
            H_kv = 1 if G == 16 else (2 if i % 2 else 1)
            B = 3 if i % 3 == 0 else 1
            cases.append((B, N, G * H_kv, H_kv, d, i % 2 == 0))
            i += 1
    return cases


@pytest.mark.parametrize("B,N,H_q,H_kv,d,causal", _sweep())
def test_fwd_shape_sweep(sqa, B, N, H_q, H_kv, d, causal):
    _check_fwd(sqa, B, N, H_q, H_kv, d, causal, seed=1000 + N + d)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_fwd_bf16_output(sqa, causal, d):
    _check_fwd(sqa, 2, 300, 8, 2, d, causal, seed=77, out_dtype=torch.bfloat16)


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_large_scores_and_custom_scale(sqa, causal):
    """Scores of magnitude ~100 exercise the running-max rescaling."""
    _check_fwd(sqa, 1, 640, 4, 4, 64, causal, seed=5, scale=1.0, mult=1.25)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_fwd_running_max_jumps(sqa, causal, d):
    """Key blocks whose scores jump by ~8-20 and by ~30-60 log2 units over
    the running max of the blocks before them: the first kind is kept
    against the stale max and moved at the next block, the second is
    recomputed in two passes from the scores."""
    N = 1024
    x = attention_inputs(1, N, 4, 2, d, seed=31 + d, device="cuda")
    k = x["k"].float()
    k[:, 256:384] *= 4.0
    k[:, 640:768] *= 12.0
    k[:, 900:1000] *= 0.25
    x["k"] = k.to(torch.bfloat16)
    o, lse = run_fwd(sqa, x["q"], x["k"], x["v"], causal)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    o_ref, lse_ref = _oracle_fwd(x, causal)
    assert_close(f64(o), o_ref, "O")
    assert_close(f64(lse), lse_ref, "LSE")


@pytest.mark.parametrize("H_q,H_kv,causal", [(6, 2, True), (12, 4, False), (6, 1, True), (24, 8, False)])
def test_fwd_group_not_power_of_two(sqa, H_q, H_kv, causal):
    """G = 3 or 6: the tile packs the largest power of two dividing G and a
    KV head's query heads span several CTAs."""
    _check_fwd(sqa, 2, 333, H_q, H_kv, 64, causal, seed=60 + H_q)


def test_fwd_mha_mqa_extremes(sqa):
    _check_fwd(sqa, 1, 384, 16, 16, 64, True, seed=9)   # MHA
    _check_fwd(sqa, 1, 384, 16, 1, 64, False, seed=10)  # MQA-style single KV head
    _check_fwd(sqa, 1, 384, 4, 1, 128, True, seed=11)   # xSMQA head counts


# ----------------------------------------------------------------------------
# Encoder-style long sequences: sampled rows against the oracle.
# ----------------------------------------------------------------------------
ENCODER_VARIANTS = [(16, 16), (16, 4), (8, 4), (8, 8), (4, 4)]


@pytest.mark.parametrize("H_q,H_kv", ENCODER_VARIANTS)
def test_encoder_32k_sampled_rows(sqa, H_q, H_kv):
    """B=1, N=32768, d=128, non-causal, seed 2; 512 seeded sampled query rows
    checked for every query head."""
    N, d = 32768, 128
    x = attention_inputs(1, N, H_q, H_kv, d, seed=2, device="cuda")
    o, lse = run_fwd(sqa, x["q"], x["k"], x["v"], False)
    sqa.sqa_device_status()
    rows = sample_rows(N, 512, seed=2)
    ri = torch.as_tensor(rows, device="cuda")
    o_ref, lse_ref = _oracle_fwd(x, False, rows=rows)
    assert_close(f64(o[:, ri]), o_ref, "O rows")
    assert_close(f64(lse[:, :, ri]), lse_ref, "LSE rows")


@pytest.mark.parametrize("N", [131072, 200000])
@pytest.mark.parametrize("H_q,H_kv", [(4, 4), (8, 4), (16, 16)])
def test_long_sequence_sampled_rows_per_head(sqa, N, H_q, H_kv):
    """B=1, d=128, non-causal, seed 3; 256 seeded rows drawn per query head."""
    d = 128
    x = attention_inputs(1, N, H_q, H_kv, d, seed=3, device="cuda")
    o, lse = run_fwd(sqa, x["q"], x["k"], x["v"], False)
    sqa.sqa_device_status()
    G = H_q // H_kv
    k_host, v_host = f64(x["k"]), f64(x["v"])
    for h in range(H_q):
        rows = sample_rows(N, 256, seed=3000 + h)
        ri = torch.as_tensor(rows, device="cuda")
        j = h // G
        q_rows = np.zeros((1, N, 1, d))
        q_rows[0, rows, 0] = f64(x["q"][0, ri, h])
        o_ref, lse_ref = attention_forward(q_rows, k_host[:, :, j:j + 1], v_host[:, :, j:j + 1], False,
                                           1 / math.sqrt(d), rows=rows)
        assert_close(f64(o[0, ri, h]), o_ref[0, :, 0], f"O head {h}")
        assert_close(f64(lse[0, h, ri]), lse_ref[0, 0], f"LSE head {h}")


@pytest.mark.parametrize("N,H_q,H_kv,boundary", [(40883, 4, 4, 148 * 2 * 128), (32768, 4, 1, 444 * 2 * 32)])
def test_mixed_grid_boundary_rows(sqa, N, H_q, H_kv, boundary):
    """Unmasked d = 128 problems whose two-tile grid leaves a mostly empty
    last wave run the two-tile kernel on the token blocks that fill whole
    waves and the split kernel on the rest (148 SMs: 40883 tokens of xSQA,
    boundary at token 37888; 32768 tokens of (4,1), four heads packed per
    tile, boundary at token 28416).  Rows on both sides of the boundary, in
    the ragged last tile and sampled elsewhere, against the oracle."""
    d = 128
    x = attention_inputs(1, N, H_q, H_kv, d, seed=41, device="cuda")
    o, lse = run_fwd(sqa, x["q"], x["k"], x["v"], False)
    sqa.sqa_device_status()
    edge = [0, 1, boundary - 2, boundary - 1, boundary, boundary + 1, N - 2, N - 1]
    rows = np.unique(np.concatenate([sample_rows(N, 96, seed=41), np.array(edge)]))
    ri = torch.as_tensor(rows, device="cuda")
    o_ref, lse_ref = _oracle_fwd(x, False, rows=rows)
    assert_close(f64(o[:, ri]), o_ref, "O rows")
    assert_close(f64(lse[:, :, ri]), lse_ref, "LSE rows")


def test_fwd_deterministic(sqa):
    x = attention_inputs(1, 1000, 8, 4, 64, seed=12, device="cuda")
    o1, l1 = run_fwd(sqa, x["q"], x["k"], x["v"], True)
    o2, l2 = run_fwd(sqa, x["q"], x["k"], x["v"], True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("H_q,H_kv,causal", [(32, 1, True), (64, 1, False), (128, 1, True), (128, 2, False)])
def test_fwd_wide_groups(sqa, H_q, H_kv, causal):
    """G = 32 .. 128 query heads per KV head: a 128-row tile packs 128 / G
    tokens (down to one token of 128 heads), the limit of the head packing."""
    _check_fwd(sqa, 1, 200, H_q, H_kv, 64, causal, seed=200 + H_q)
