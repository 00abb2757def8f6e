"""GPU parity of KV-cache decoding against the fp64 oracle: ragged cache
lengths, one or several new tokens per sequence, the head-count variants,
one-chunk and multi-chunk (split + combine) plans, bf16 output, and a cache
length out of range reported by the device status word."""

import math

import numpy as np
import pytest
import torch

from oracle import attention_decode
from parity import assert_close, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sqa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_query_attention_b200 as lib
    return lib


def _inputs(B, n_new, H_q, H_kv, d, L_max, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    draw = lambda shape: torch.randn(shape, generator=g, device="cuda").to(torch.bfloat16)
    return draw((B, n_new, H_q, d)), draw((B, L_max, H_kv, d)), draw((B, L_max, H_kv, d))


def _decode(sqa, q, kc, vc, lens, out_dtype=torch.float32, with_lse=True):
    B, n_new, H_q, d = q.shape
    L_max, H_kv = kc.shape[1], kc.shape[2]
    out = torch.empty((B, n_new, H_q, d), dtype=out_dtype, device="cuda")
    lse = torch.empty((B, H_q, n_new), dtype=torch.float32, device="cuda") if with_lse else None
    wsb = sqa.sqa_attn_decode_workspace_size(B, n_new, H_q, H_kv, d, L_max)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda")
    dt = sqa.SQA_DT_BF16 if out_dtype == torch.bfloat16 else sqa.SQA_DT_F32
    lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    sqa.sqa_attn_decode(q, kc, vc, lens_d, out, dt, lse, B, n_new, H_q, H_kv, d, L_max, 1 / math.sqrt(d),
                        ws if wsb else None, wsb)
    return out, lse


CASES = [
    # B, n_new, H_q, H_kv, d, L_max, lens
    (4, 1, 8, 4, 128, 4096, [4096, 1, 1000, 2049]),      # SQA, ragged, multi-chunk
    (2, 4, 8, 4, 64, 3000, [3000, 4]),                    # four new tokens (causal among them)
    (3, 1, 16, 1, 64, 2500, [2500, 777, 129]),            # G = 16 in one tile
    (2, 2, 6, 2, 128, 1500, [1500, 64]),                  # G = 3: three head sub-groups
    (1, 1, 16, 16, 128, 9000, [8999]),                    # MHA head count
    (5, 1, 4, 4, 32, 200, [200, 1, 64, 65, 199]),         # one chunk per sequence
    (2, 16, 8, 1, 16, 700, [700, 16]),                    # 8 heads x 16 tokens = 128 rows
]


@pytest.mark.parametrize("B,n_new,H_q,H_kv,d,L_max,lens", CASES)
def test_decode_matches_oracle(sqa, B, n_new, H_q, H_kv, d, L_max, lens):
    q, kc, vc = _inputs(B, n_new, H_q, H_kv, d, L_max, seed=L_max + n_new)
    o, lse = _decode(sqa, q, kc, vc, lens)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    ro, rl = attention_decode(f64(q), f64(kc), f64(vc), np.asarray(lens), 1 / math.sqrt(d))
    assert_close(f64(o), ro, "O")
    assert_close(f64(lse), rl, "LSE")


def test_decode_large_cache_bf16_out(sqa):
    """B=8 sequences of up to 32768 cached tokens, SQA (8, 4), d=128, bf16
    output; cache entries past each length hold NaN and are never read."""
    B, n_new, H_q, H_kv, d, L_max = 8, 1, 8, 4, 128, 32768
    lens = [32768, 30000, 17, 12345, 32767, 1, 8192, 20000]
    q, kc, vc = _inputs(B, n_new, H_q, H_kv, d, L_max, seed=77)
    for b, L in enumerate(lens):
        kc[b, L:] = float("nan")
        vc[b, L:] = float("nan")
    o, lse = _decode(sqa, q, kc, vc, lens, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    ro, rl = attention_decode(f64(q), f64(kc), f64(vc), np.asarray(lens), 1 / math.sqrt(d))
    assert_close(f64(o), ro, "O")
    assert_close(f64(lse), rl, "LSE")


def test_decode_bad_length_is_reported(sqa):
    """A cache length past L_max is clamped in the kernel (no access past the
    cache) and reported once by sqa_device_status as SQA_ERR_INVALID_ARG."""
    B, n_new, H_q, H_kv, d, L_max = 2, 1, 4, 2, 64, 512
    q, kc, vc = _inputs(B, n_new, H_q, H_kv, d, L_max, seed=3)
    o, _ = _decode(sqa, q, kc, vc, [L_max + 100, 10])
    with pytest.raises(sqa.SQAError) as e:
        sqa.sqa_device_status()
    assert e.value.status == sqa.SQA_ERR_INVALID_ARG
    sqa.sqa_device_status()  # cleared
    ro, _ = attention_decode(f64(q), f64(kc), f64(vc), np.asarray([L_max, 10]), 1 / math.sqrt(d))
    assert_close(f64(o), ro, "O (clamped length)")


def test_decode_bench_configuration(sqa):
    """The benchmark's decode step exactly: B=16 sequences with 32768 cached
    tokens each, SQA (8, 4), d=128, one new token, bf16 output (18 chunks of
    1856 keys per sequence and KV head, merged by the combine pass)."""
    B, n_new, H_q, H_kv, d, L_max = 16, 1, 8, 4, 128, 32768
    assert sqa.sqa_attn_decode_workspace_size(B, n_new, H_q, H_kv, d, L_max) > 0
    q, kc, vc = _inputs(B, n_new, H_q, H_kv, d, L_max, seed=5)
    o, lse = _decode(sqa, q, kc, vc, [L_max] * B, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    sqa.sqa_device_status()
    ro, rl = attention_decode(f64(q), f64(kc), f64(vc), np.full(B, L_max), 1 / math.sqrt(d))
    assert_close(f64(o), ro, "O")
    assert_close(f64(lse), rl, "LSE")
