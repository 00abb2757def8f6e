"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, and rejects invalid arguments before launching anything."""

import ctypes
import os
import re

import pytest

import sparse_query_attention_b200 as sqa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sqa.h")

FAKE = 0x10000  # a 16-byte-aligned non-null address; never dereferenced here


def _declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sqa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_expected_entry_points():
    names = _declared_symbols()
    for n in ("sqa_attn_fwd", "sqa_attn_fwd_ex", "sqa_attn_bwd", "sqa_attn_bwd_workspace_size",
              "sqa_attn_fwd_cross", "sqa_attn_bwd_cross", "sqa_attn_fwd_packed", "sqa_attn_bwd_packed",
              "sqa_attn_fwd_window", "sqa_attn_bwd_window", "sqa_attn_decode", "sqa_attn_decode_workspace_size",
              "sqa_proj", "sqa_device_status", "sqa_status_string", "sqa_version"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(sqa.LIB_PATH)
    for name in _declared_symbols():
        assert hasattr(lib, name), name
        assert name in sqa.SIGNATURES, name


def test_status_strings_and_version():
    assert sqa.status_string(0) == "SQA_OK"
    assert sqa.status_string(4) == "SQA_ERR_TIMEOUT"
    assert sqa.status_string(99) == "SQA_ERR_UNKNOWN"
    assert re.fullmatch(r"\d+\.\d+\.\d+", sqa.sqa_version())


def _fwd(**kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, B=1, N=8, H_q=4, H_kv=2, d=32, causal=1, scale=0.17)
    args.update(kw)
    return sqa.library().sqa_attn_fwd(args["q"], args["k"], args["v"], args["out"], args["B"], args["N"],
                                      args["H_q"], args["H_kv"], args["d"], args["causal"], args["scale"], None)


@pytest.mark.parametrize("kw", [
    dict(q=None), dict(k=None), dict(v=None), dict(out=None),
    dict(B=0), dict(N=0), dict(N=-3), dict(H_q=0), dict(H_kv=0),
    dict(H_q=4, H_kv=3), dict(H_q=2, H_kv=4), dict(scale=float("inf")), dict(scale=float("nan")),
    dict(q=FAKE + 8), dict(out=FAKE + 4), dict(d=0),
])
def test_fwd_rejects_invalid_arguments(kw):
    assert _fwd(**kw) == sqa.SQA_ERR_INVALID_ARG


@pytest.mark.parametrize("d", [8, 48, 96, 256])
def test_fwd_rejects_unsupported_head_dim(d):
    assert _fwd(d=d) == sqa.SQA_ERR_UNSUPPORTED


def test_fwd_ex_rejects_bad_dtype_and_lse_alignment():
    lib = sqa.library()
    assert lib.sqa_attn_fwd_ex(FAKE, FAKE, FAKE, FAKE, 7, None, 1, 8, 4, 2, 32, 1, 0.1, None) == sqa.SQA_ERR_INVALID_ARG
    assert lib.sqa_attn_fwd_ex(FAKE, FAKE, FAKE, FAKE, 0, FAKE + 4, 1, 8, 4, 2, 32, 1, 0.1, None) == sqa.SQA_ERR_INVALID_ARG


def test_bwd_workspace_size():
    assert sqa.sqa_attn_bwd_workspace_size(4, 8192, 8, 4, 64) >= 4 * 8 * 8192 * 4
    assert sqa.sqa_attn_bwd_workspace_size(4, 8192, 8, 4, 64) % 256 == 0
    assert sqa.sqa_attn_bwd_workspace_size(0, 8, 8, 4, 64) == 0
    assert sqa.sqa_attn_bwd_workspace_size(1, 8, 6, 4, 64) == 0


def test_bwd_rejects_invalid_arguments():
    lib = sqa.library()
    ws = sqa.sqa_attn_bwd_workspace_size(1, 8, 4, 2, 32)

    def call(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, od=0, do=FAKE, lse=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, gd=0,
                 B=1, N=8, H_q=4, H_kv=2, d=32, causal=1, scale=0.2, ws=FAKE, wsb=ws)
        a.update(kw)
        return lib.sqa_attn_bwd(a["q"], a["k"], a["v"], a["o"], a["od"], a["do"], a["lse"], a["dq"], a["dk"],
                                a["dv"], a["gd"], a["B"], a["N"], a["H_q"], a["H_kv"], a["d"], a["causal"],
                                a["scale"], a["ws"], a["wsb"], None)

    for kw in (dict(do=None), dict(lse=None), dict(dk=None), dict(ws=None), dict(wsb=ws - 4),
               dict(od=5), dict(gd=2), dict(H_kv=3), dict(dq=FAKE + 2)):
        assert call(**kw) == sqa.SQA_ERR_INVALID_ARG, kw
    assert call(d=80) == sqa.SQA_ERR_UNSUPPORTED


def test_cross_rejects_invalid_lengths():
    lib = sqa.library()
    for n_q, n_kv in ((0, 8), (8, 0), (8, -1)):
        assert lib.sqa_attn_fwd_cross(FAKE, FAKE, FAKE, FAKE, 0, None, 1, n_q, n_kv, 4, 2, 32, 0.1,
                                      None) == sqa.SQA_ERR_INVALID_ARG
    ws = sqa.sqa_attn_bwd_workspace_size(1, 8, 4, 2, 32)
    assert lib.sqa_attn_bwd_cross(FAKE, FAKE, FAKE, FAKE, 0, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 1, 8, 0, 4, 2, 32,
                                  0.1, FAKE, ws, None) == sqa.SQA_ERR_INVALID_ARG
    # The workspace holds per-query-row values: sized for N_q, not N_kv.
    assert lib.sqa_attn_bwd_cross(FAKE, FAKE, FAKE, FAKE, 0, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 1, 4096, 8, 4, 2, 32,
                                  0.1, FAKE, ws, None) == sqa.SQA_ERR_INVALID_ARG


def test_window_rejects_invalid_arguments():
    lib = sqa.library()
    for left, right in ((-1, 0), (0, -1), (-5, -5)):
        assert lib.sqa_attn_fwd_window(FAKE, FAKE, FAKE, FAKE, 0, None, 1, 8, 4, 2, 32, left, right, 0.1,
                                       None) == sqa.SQA_ERR_INVALID_ARG
    assert lib.sqa_attn_fwd_window(FAKE, FAKE, FAKE, FAKE, 0, None, 1, 0, 4, 2, 32, 3, 0, 0.1,
                                   None) == sqa.SQA_ERR_INVALID_ARG
    ws = sqa.sqa_attn_bwd_workspace_size(1, 8, 4, 2, 32)
    assert lib.sqa_attn_bwd_window(FAKE, FAKE, FAKE, FAKE, 0, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 1, 8, 4, 2, 32,
                                   -1, 0, 0.1, FAKE, ws, None) == sqa.SQA_ERR_INVALID_ARG
    assert lib.sqa_attn_bwd_window(FAKE, FAKE, FAKE, FAKE, 0, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 1, 8, 4, 2, 32,
                                   2, 2, 0.1, FAKE, ws - 4, None) == sqa.SQA_ERR_INVALID_ARG


def test_decode_workspace_and_invalid_arguments():
    lib = sqa.library()
    # One chunk per sequence (L_max <= 256): no workspace.
    assert sqa.sqa_attn_decode_workspace_size(4, 1, 8, 4, 128, 256) == 0
    ws = sqa.sqa_attn_decode_workspace_size(2, 1, 8, 4, 128, 32768)
    assert ws > 0 and ws % 16 == 0
    assert sqa.sqa_attn_decode_workspace_size(2, 4, 8, 3, 128, 100) == 0
    assert sqa.sqa_attn_decode_workspace_size(2, 8, 8, 4, 128, 4) == 0   # L_max < n_new

    def call(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, lens=FAKE, out=FAKE, od=0, lse=None, B=2, n=1, H_q=8, H_kv=4, d=128,
                 L=32768, scale=0.1, ws=FAKE, wsb=ws)
        a.update(kw)
        return lib.sqa_attn_decode(a["q"], a["k"], a["v"], a["lens"], a["out"], a["od"], a["lse"], a["B"], a["n"],
                                   a["H_q"], a["H_kv"], a["d"], a["L"], a["scale"], a["ws"], a["wsb"], None)

    for kw in (dict(lens=None), dict(out=None), dict(ws=None), dict(wsb=ws - 16), dict(od=4), dict(n=0),
               dict(L=0), dict(H_kv=3), dict(lens=FAKE + 2), dict(out=FAKE + 8)):
        assert call(**kw) == sqa.SQA_ERR_INVALID_ARG, kw
    assert call(d=96) == sqa.SQA_ERR_UNSUPPORTED
    # 2 heads per group x 65 new tokens = 130 rows > one 128-row tile.
    assert call(n=65, wsb=1 << 30) == sqa.SQA_ERR_UNSUPPORTED


def test_size_limits_are_rejected_before_launch():
    """Shapes past the kernels' 32-bit index ranges return
    SQA_ERR_UNSUPPORTED from the host checks (nothing is launched, so fake
    pointers are safe here)."""
    lib = sqa.library()
    # B * N * H_q rows at 2^31.
    assert _fwd(B=1, N=1 << 28, H_q=8, H_kv=4, causal=0) == sqa.SQA_ERR_UNSUPPORTED
    assert _fwd(B=2, N=1 << 27, H_q=8, H_kv=8, causal=0) == sqa.SQA_ERR_UNSUPPORTED
    # A band (causal or window) needs N <= 2^30.
    assert lib.sqa_attn_fwd_window(FAKE, FAKE, FAKE, FAKE, 0, None, 1, (1 << 30) + 64, 1, 1, 32, 5, 0, 0.1,
                                   None) == sqa.SQA_ERR_UNSUPPORTED
    # Key rows B * N_kv * H_kv at 2^31 for cross attention.
    assert lib.sqa_attn_fwd_cross(FAKE, FAKE, FAKE, FAKE, 0, None, 1, 16, 1 << 29, 4, 4, 32, 0.1,
                                  None) == sqa.SQA_ERR_UNSUPPORTED
    # Decode caches of B * L_max * H_kv >= 2^31 rows.
    ws = sqa.sqa_attn_decode_workspace_size(2, 1, 8, 8, 64, 1 << 27)
    assert lib.sqa_attn_decode(FAKE, FAKE, FAKE, FAKE, FAKE, 0, None, 2, 1, 8, 8, 64, 1 << 27, 0.1, FAKE, ws,
                               None) == sqa.SQA_ERR_UNSUPPORTED


def test_packed_rejects_invalid_arguments():
    lib = sqa.library()
    assert lib.sqa_attn_fwd_packed(None, FAKE, 0, None, 1, 8, 4, 2, 32, 1, 0.1, None) == sqa.SQA_ERR_INVALID_ARG
    assert lib.sqa_attn_fwd_packed(FAKE, FAKE, 0, None, 1, 8, 4, 3, 32, 1, 0.1, None) == sqa.SQA_ERR_INVALID_ARG
    assert lib.sqa_attn_fwd_packed(FAKE, FAKE, 0, None, 1, 8, 4, 0, 32, 1, 0.1, None) == sqa.SQA_ERR_INVALID_ARG
    assert lib.sqa_attn_fwd_packed(FAKE, FAKE, 0, None, 1, 8, 4, 2, 48, 1, 0.1, None) == sqa.SQA_ERR_UNSUPPORTED
    ws = sqa.sqa_attn_bwd_workspace_size(1, 8, 4, 2, 32)
    assert lib.sqa_attn_bwd_packed(FAKE, FAKE, 0, FAKE, FAKE, None, 0, 1, 8, 4, 2, 32, 1, 0.1, FAKE, ws,
                                   None) == sqa.SQA_ERR_INVALID_ARG
    assert lib.sqa_attn_bwd_packed(FAKE, FAKE, 0, FAKE, FAKE, FAKE, 9, 1, 8, 4, 2, 32, 1, 0.1, FAKE, ws,
                                   None) == sqa.SQA_ERR_INVALID_ARG


def test_proj_rejects_invalid_arguments():
    lib = sqa.library()
    assert lib.sqa_proj(None, FAKE, None, FAKE, 0, 128, 64, 64, None) == sqa.SQA_ERR_INVALID_ARG
    assert lib.sqa_proj(FAKE, FAKE, None, FAKE, 0, 0, 64, 64, None) == sqa.SQA_ERR_INVALID_ARG
    assert lib.sqa_proj(FAKE, FAKE, None, FAKE, 3, 128, 64, 64, None) == sqa.SQA_ERR_INVALID_ARG
    assert lib.sqa_proj(FAKE, FAKE, FAKE + 4, FAKE, 0, 128, 64, 64, None) == sqa.SQA_ERR_INVALID_ARG
    assert lib.sqa_proj(FAKE, FAKE, None, FAKE, 0, 128, 40, 64, None) == sqa.SQA_ERR_UNSUPPORTED
    assert lib.sqa_proj(FAKE, FAKE, None, FAKE, 0, 128, 64, 24, None) == sqa.SQA_ERR_UNSUPPORTED


def test_selftest_rejects_out_of_range_timeout():
    lib = sqa.library()
    assert lib.sqa_selftest_wait_timeout(0, None) == sqa.SQA_ERR_INVALID_ARG
    assert lib.sqa_selftest_wait_timeout(20000, None) == sqa.SQA_ERR_INVALID_ARG


def test_binding_raises_on_error_status():
    with pytest.raises(sqa.SQAError) as e:
        sqa.sqa_attn_fwd(FAKE, FAKE, FAKE, FAKE, 1, 8, 4, 3, 32, True, 0.1, stream=0)
    assert e.value.status == sqa.SQA_ERR_INVALID_ARG


def test_binding_checks_tensor_dtype_and_size():
    """The binding rejects tensors of the wrong element type or too few
    elements before calling the library (CPU tensors reach these checks
    first; a CUDA tensor is needed only to get past them)."""
    import torch
    q = torch.zeros(2 * 8 * 4 * 32, dtype=torch.float32)
    with pytest.raises(ValueError, match="expected torch.bfloat16"):
        sqa.sqa_attn_fwd(q, FAKE, FAKE, FAKE, 2, 8, 4, 2, 32, True, 0.1, stream=0)
    small = torch.zeros(10, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="elements"):
        sqa.sqa_attn_fwd(small, FAKE, FAKE, FAKE, 2, 8, 4, 2, 32, True, 0.1, stream=0)
    lens = torch.zeros(3, dtype=torch.int64)
    with pytest.raises(ValueError, match="expected torch.int32"):
        sqa.sqa_attn_decode(FAKE, FAKE, FAKE, lens, FAKE, 0, None, 3, 1, 4, 2, 32, 64, 0.1, None, 0, stream=0)
