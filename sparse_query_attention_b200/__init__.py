"""Python binding of libsqa.so, the B200 (sm_100a) Sparse Query Attention hot path.

Each function has the name and argument order of the C entry point in
``include/sqa.h`` and only marshals arguments: tensors become raw device
pointers, ``stream=None`` becomes torch's current CUDA stream, and a non-OK
status raises :class:`SQAError`.  Every step of the computation runs in the
library's CUDA kernels; there is no other implementation behind these names.

The library must have been built (``python -m sparse_query_attention_b200.build``);
the first call into it raises ImportError when it is missing.
"""

from __future__ import annotations

import ctypes
import os

from .build import LIB_PATH

SQA_OK = 0
SQA_ERR_INVALID_ARG = 1
SQA_ERR_UNSUPPORTED = 2
SQA_ERR_CUDA = 3
SQA_ERR_TIMEOUT = 4

SQA_DT_F32 = 0
SQA_DT_BF16 = 1

SQA_K_CONTIGUOUS = 0
SQA_MN_CONTIGUOUS = 1

# Every symbol include/sqa.h declares, with (restype, argtypes).
_P, _I, _F, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "sqa_attn_fwd": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "sqa_attn_fwd_ex": (_I, [_P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "sqa_attn_fwd_cross": (_I, [_P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "sqa_attn_fwd_window": (_I, [_P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P]),
    "sqa_attn_decode_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I]),
    "sqa_attn_decode": (_I, [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _F, _P, _Z, _P]),
    "sqa_attn_fwd_packed": (_I, [_P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _F, _P]),
    "sqa_attn_bwd_workspace_size": (_Z, [_I, _I, _I, _I, _I]),
    "sqa_attn_bwd": (_I, [_P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _I,
                          _I, _I, _I, _I, _I, _I, _F, _P, _Z, _P]),
    "sqa_attn_bwd_cross": (_I, [_P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _I,
                                _I, _I, _I, _I, _I, _I, _F, _P, _Z, _P]),
    "sqa_attn_bwd_window": (_I, [_P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _I,
                                 _I, _I, _I, _I, _I, _I, _I, _F, _P, _Z, _P]),
    "sqa_attn_bwd_packed": (_I, [_P, _P, _I, _P, _P, _P, _I,
                                 _I, _I, _I, _I, _I, _I, _F, _P, _Z, _P]),
    "sqa_attn_bwd_static": (_I, [_P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _I,
                                 _I, _I, _I, _I, _I, _I, _F, _P]),
    "sqa_proj": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "sqa_gemm": (_I, [_P, _I, _P, _I, _P, _P, _I, _I, _I, _I, _I, _P]),
    "sqa_device_status": (_I, [_P]),
    "sqa_selftest_wait_timeout": (_I, [_I, _P]),
    "sqa_status_string": (ctypes.c_char_p, [_I]),
    "sqa_version": (ctypes.c_char_p, []),
}


class SQAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing; build it with `python -m sparse_query_attention_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_handle = None


def library() -> ctypes.CDLL:
    """The loaded libsqa.so (loaded on first use; raises ImportError if it
    has not been built)."""
    global _handle
    if _handle is None:
        _handle = _load()
    return _handle


def _ptr(x):
    """Device pointer of a CUDA tensor (or an int / None passed through)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not x.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not x.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str) -> None:
    if status != SQA_OK:
        raise SQAError(status, where)


def status_string(status: int) -> str:
    return library().sqa_status_string(int(status)).decode()


def sqa_version() -> str:
    return library().sqa_version().decode()


def sqa_status_string(status: int) -> str:
    return status_string(status)


_BF, _F32, _I32, _U8 = "torch.bfloat16", "torch.float32", "torch.int32", "torch.uint8"
_DT = {SQA_DT_F32: _F32, SQA_DT_BF16: _BF}


def _t(x, dtype, numel, name):
    """_ptr with the checks the C ABI cannot make: a torch tensor must have
    the element type the call reads or writes and at least the elements the
    shape arguments imply (integers and None pass through unchecked)."""
    if x is not None and not isinstance(x, int):
        if dtype is not None and str(x.dtype) != dtype:
            raise ValueError(f"{name}: expected {dtype}, got {x.dtype}")
        if numel > 0 and x.numel() < numel:
            raise ValueError(f"{name}: {x.numel()} elements, the shape needs {numel}")
    return _ptr(x)


def sqa_attn_fwd(q, k, v, out, B, N, H_q, H_kv, d_head, causal, scale, stream=None) -> None:
    nq, nkv = B * N * H_q * d_head, B * N * H_kv * d_head
    _check(library().sqa_attn_fwd(_t(q, _BF, nq, "q"), _t(k, _BF, nkv, "k"), _t(v, _BF, nkv, "v"),
                                  _t(out, _F32, nq, "out"), B, N, H_q, H_kv, d_head, int(bool(causal)),
                                  float(scale), _stream(stream)), "sqa_attn_fwd")


def sqa_attn_fwd_ex(q, k, v, out, out_dtype, lse, B, N, H_q, H_kv, d_head, causal, scale,
                    stream=None) -> None:
    nq, nkv = B * N * H_q * d_head, B * N * H_kv * d_head
    _check(library().sqa_attn_fwd_ex(_t(q, _BF, nq, "q"), _t(k, _BF, nkv, "k"), _t(v, _BF, nkv, "v"),
                                     _t(out, _DT.get(out_dtype), nq, "out"), int(out_dtype),
                                     _t(lse, _F32, B * H_q * N, "lse"), B, N, H_q, H_kv, d_head, int(bool(causal)),
                                     float(scale), _stream(stream)), "sqa_attn_fwd_ex")


def sqa_attn_fwd_cross(q, k, v, out, out_dtype, lse, B, N_q, N_kv, H_q, H_kv, d_head, scale,
                       stream=None) -> None:
    """Cross / memory attention: N_q queries, N_kv keys, no mask."""
    nq, nkv = B * N_q * H_q * d_head, B * N_kv * H_kv * d_head
    _check(library().sqa_attn_fwd_cross(_t(q, _BF, nq, "q"), _t(k, _BF, nkv, "k"), _t(v, _BF, nkv, "v"),
                                        _t(out, _DT.get(out_dtype), nq, "out"), int(out_dtype),
                                        _t(lse, _F32, B * H_q * N_q, "lse"), B, N_q, N_kv, H_q, H_kv, d_head,
                                        float(scale), _stream(stream)), "sqa_attn_fwd_cross")


def sqa_attn_fwd_window(q, k, v, out, out_dtype, lse, B, N, H_q, H_kv, d_head, window_left, window_right,
                        scale, stream=None) -> None:
    """Sliding-window forward: query t sees keys t - left .. t + right."""
    nq, nkv = B * N * H_q * d_head, B * N * H_kv * d_head
    _check(library().sqa_attn_fwd_window(_t(q, _BF, nq, "q"), _t(k, _BF, nkv, "k"), _t(v, _BF, nkv, "v"),
                                         _t(out, _DT.get(out_dtype), nq, "out"), int(out_dtype),
                                         _t(lse, _F32, B * H_q * N, "lse"), B, N, H_q, H_kv, d_head,
                                         int(window_left), int(window_right), float(scale), _stream(stream)),
           "sqa_attn_fwd_window")


def sqa_attn_decode_workspace_size(B, n_new, H_q, H_kv, d_head, L_max) -> int:
    return int(library().sqa_attn_decode_workspace_size(B, n_new, H_q, H_kv, d_head, L_max))


def sqa_attn_decode(q, k_cache, v_cache, cache_lens, out, out_dtype, lse, B, n_new, H_q, H_kv, d_head, L_max,
                    scale, workspace, workspace_bytes, stream=None) -> None:
    """Decode n_new tokens per sequence against a KV cache; cache_lens is a
    device int32 tensor [B]."""
    nq, nc = B * n_new * H_q * d_head, B * L_max * H_kv * d_head
    _check(library().sqa_attn_decode(_t(q, _BF, nq, "q"), _t(k_cache, _BF, nc, "k_cache"),
                                     _t(v_cache, _BF, nc, "v_cache"), _t(cache_lens, _I32, B, "cache_lens"),
                                     _t(out, _DT.get(out_dtype), nq, "out"), int(out_dtype),
                                     _t(lse, _F32, B * H_q * n_new, "lse"), B, n_new, H_q, H_kv, d_head, L_max,
                                     float(scale), _t(workspace, _U8, int(workspace_bytes), "workspace"),
                                     int(workspace_bytes), _stream(stream)), "sqa_attn_decode")


def sqa_attn_fwd_packed(qkv, out, out_dtype, lse, B, N, H_q, H_kv, d_head, causal, scale,
                        stream=None) -> None:
    """Forward on a packed QKV buffer [B, N, H_q + 2*H_kv, d_head]."""
    _check(library().sqa_attn_fwd_packed(_t(qkv, _BF, B * N * (H_q + 2 * H_kv) * d_head, "qkv"),
                                         _t(out, _DT.get(out_dtype), B * N * H_q * d_head, "out"), int(out_dtype),
                                         _t(lse, _F32, B * H_q * N, "lse"), B, N, H_q, H_kv, d_head,
                                         int(bool(causal)), float(scale), _stream(stream)), "sqa_attn_fwd_packed")


def sqa_attn_bwd_workspace_size(B, N, H_q, H_kv, d_head) -> int:
    return int(library().sqa_attn_bwd_workspace_size(B, N, H_q, H_kv, d_head))


def _bwd_args(q, k, v, out, o_dtype, dout, lse, dq, dk, dv, grad_dtype, B, N_q, N_kv, H_q, H_kv, d_head):
    nq, nkv = B * N_q * H_q * d_head, B * N_kv * H_kv * d_head
    g = _DT.get(grad_dtype)
    return (_t(q, _BF, nq, "q"), _t(k, _BF, nkv, "k"), _t(v, _BF, nkv, "v"), _t(out, _DT.get(o_dtype), nq, "out"),
            int(o_dtype), _t(dout, _BF, nq, "dout"), _t(lse, _F32, B * H_q * N_q, "lse"), _t(dq, g, nq, "dq"),
            _t(dk, g, nkv, "dk"), _t(dv, g, nkv, "dv"), int(grad_dtype))


def sqa_attn_bwd(q, k, v, out, o_dtype, dout, lse, dq, dk, dv, grad_dtype, B, N, H_q, H_kv,
                 d_head, causal, scale, workspace, workspace_bytes, stream=None) -> None:
    _check(library().sqa_attn_bwd(*_bwd_args(q, k, v, out, o_dtype, dout, lse, dq, dk, dv, grad_dtype, B, N, N,
                                             H_q, H_kv, d_head),
                                  B, N, H_q, H_kv, d_head, int(bool(causal)), float(scale),
                                  _t(workspace, _U8, int(workspace_bytes), "workspace"), int(workspace_bytes),
                                  _stream(stream)), "sqa_attn_bwd")


def sqa_attn_bwd_cross(q, k, v, out, o_dtype, dout, lse, dq, dk, dv, grad_dtype, B, N_q, N_kv, H_q,
                       H_kv, d_head, scale, workspace, workspace_bytes, stream=None) -> None:
    """Gradient of sqa_attn_fwd_cross; workspace sized for N_q query rows."""
    _check(library().sqa_attn_bwd_cross(*_bwd_args(q, k, v, out, o_dtype, dout, lse, dq, dk, dv, grad_dtype, B,
                                                   N_q, N_kv, H_q, H_kv, d_head),
                                        B, N_q, N_kv, H_q, H_kv, d_head, float(scale),
                                        _t(workspace, _U8, int(workspace_bytes), "workspace"), int(workspace_bytes),
                                        _stream(stream)), "sqa_attn_bwd_cross")


def sqa_attn_bwd_window(q, k, v, out, o_dtype, dout, lse, dq, dk, dv, grad_dtype, B, N, H_q, H_kv, d_head,
                        window_left, window_right, scale, workspace, workspace_bytes, stream=None) -> None:
    """Gradient of sqa_attn_fwd_window (same window)."""
    _check(library().sqa_attn_bwd_window(*_bwd_args(q, k, v, out, o_dtype, dout, lse, dq, dk, dv, grad_dtype, B,
                                                    N, N, H_q, H_kv, d_head),
                                         B, N, H_q, H_kv, d_head, int(window_left), int(window_right),
                                         float(scale), _t(workspace, _U8, int(workspace_bytes), "workspace"),
                                         int(workspace_bytes), _stream(stream)), "sqa_attn_bwd_window")


def sqa_attn_bwd_packed(qkv, out, o_dtype, dout, lse, dqkv, grad_dtype, B, N, H_q, H_kv, d_head, causal,
                        scale, workspace, workspace_bytes, stream=None) -> None:
    """Gradient of sqa_attn_fwd_packed into a packed dQKV buffer."""
    nq, npk = B * N * H_q * d_head, B * N * (H_q + 2 * H_kv) * d_head
    _check(library().sqa_attn_bwd_packed(_t(qkv, _BF, npk, "qkv"), _t(out, _DT.get(o_dtype), nq, "out"),
                                         int(o_dtype), _t(dout, _BF, nq, "dout"), _t(lse, _F32, B * H_q * N, "lse"),
                                         _t(dqkv, _DT.get(grad_dtype), npk, "dqkv"), int(grad_dtype),
                                         B, N, H_q, H_kv, d_head, int(bool(causal)), float(scale),
                                         _t(workspace, _U8, int(workspace_bytes), "workspace"), int(workspace_bytes),
                                         _stream(stream)), "sqa_attn_bwd_packed")


def sqa_attn_bwd_static(q, k, v, out, o_dtype, dout, lse, dq, dk, dv, grad_dtype, B, N, H_q, H_kv,
                        d_head, causal, scale, stream=None) -> None:
    """sqa_attn_bwd with the library's fixed device scratch instead of a
    caller workspace, for callers that cannot allocate device memory; see
    include/sqa.h for its size limit and sharing rules."""
    _check(library().sqa_attn_bwd_static(*_bwd_args(q, k, v, out, o_dtype, dout, lse, dq, dk, dv, grad_dtype, B,
                                                    N, N, H_q, H_kv, d_head),
                                         B, N, H_q, H_kv, d_head, int(bool(causal)), float(scale),
                                         _stream(stream)), "sqa_attn_bwd_static")


def sqa_proj(x, w, bias, y, y_dtype, M, K, Nout, stream=None) -> None:
    _check(library().sqa_proj(_t(x, _BF, M * K, "x"), _t(w, _BF, Nout * K, "w"), _t(bias, _F32, Nout, "bias"),
                              _t(y, _DT.get(y_dtype), M * Nout, "y"), int(y_dtype), M, K, Nout, _stream(stream)),
           "sqa_proj")


def sqa_gemm(a, a_layout, b, b_layout, bias, c, c_dtype, accumulate, M, N, K, stream=None) -> None:
    _check(library().sqa_gemm(_t(a, _BF, M * K, "a"), int(a_layout), _t(b, _BF, N * K, "b"), int(b_layout),
                              _t(bias, _F32, N, "bias"), _t(c, _DT.get(c_dtype), M * N, "c"), int(c_dtype),
                              int(bool(accumulate)), M, N, K, _stream(stream)), "sqa_gemm")


def sqa_device_status(stream=None) -> None:
    _check(library().sqa_device_status(_stream(stream)), "sqa_device_status")


def sqa_selftest_wait_timeout(timeout_ms, stream=None) -> None:
    _check(library().sqa_selftest_wait_timeout(int(timeout_ms), _stream(stream)), "sqa_selftest_wait_timeout")
