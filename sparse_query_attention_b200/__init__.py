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


def sqa_attn_fwd(q, k, v, out, B, N, H_q, H_kv, d_head, causal, scale, stream=None) -> None:
    _check(library().sqa_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, N, H_q, H_kv, d_head,
                             int(bool(causal)), float(scale), _stream(stream)), "sqa_attn_fwd")


def sqa_attn_fwd_ex(q, k, v, out, out_dtype, lse, B, N, H_q, H_kv, d_head, causal, scale,
                    stream=None) -> None:
    _check(library().sqa_attn_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), int(out_dtype), _ptr(lse),
                                B, N, H_q, H_kv, d_head, int(bool(causal)), float(scale),
                                _stream(stream)), "sqa_attn_fwd_ex")


def sqa_attn_fwd_cross(q, k, v, out, out_dtype, lse, B, N_q, N_kv, H_q, H_kv, d_head, scale,
                       stream=None) -> None:
    """Cross / memory attention: N_q queries, N_kv keys, no mask."""
    _check(library().sqa_attn_fwd_cross(_ptr(q), _ptr(k), _ptr(v), _ptr(out), int(out_dtype), _ptr(lse),
                                        B, N_q, N_kv, H_q, H_kv, d_head, float(scale),
                                        _stream(stream)), "sqa_attn_fwd_cross")


def sqa_attn_fwd_window(q, k, v, out, out_dtype, lse, B, N, H_q, H_kv, d_head, window_left, window_right,
                        scale, stream=None) -> None:
    """Sliding-window forward: query t sees keys t - left .. t + right."""
    _check(library().sqa_attn_fwd_window(_ptr(q), _ptr(k), _ptr(v), _ptr(out), int(out_dtype), _ptr(lse),
                                         B, N, H_q, H_kv, d_head, int(window_left), int(window_right),
                                         float(scale), _stream(stream)), "sqa_attn_fwd_window")


def sqa_attn_decode_workspace_size(B, n_new, H_q, H_kv, d_head, L_max) -> int:
    return int(library().sqa_attn_decode_workspace_size(B, n_new, H_q, H_kv, d_head, L_max))


def sqa_attn_decode(q, k_cache, v_cache, cache_lens, out, out_dtype, lse, B, n_new, H_q, H_kv, d_head, L_max,
                    scale, workspace, workspace_bytes, stream=None) -> None:
    """Decode n_new tokens per sequence against a KV cache; cache_lens is a
    device int32 tensor [B]."""
    _check(library().sqa_attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_lens), _ptr(out),
                                     int(out_dtype), _ptr(lse), B, n_new, H_q, H_kv, d_head, L_max, float(scale),
                                     _ptr(workspace), int(workspace_bytes), _stream(stream)), "sqa_attn_decode")


def sqa_attn_fwd_packed(qkv, out, out_dtype, lse, B, N, H_q, H_kv, d_head, causal, scale,
                        stream=None) -> None:
    """Forward on a packed QKV buffer [B, N, H_q + 2*H_kv, d_head]."""
    _check(library().sqa_attn_fwd_packed(_ptr(qkv), _ptr(out), int(out_dtype), _ptr(lse), B, N, H_q, H_kv,
                                         d_head, int(bool(causal)), float(scale), _stream(stream)),
           "sqa_attn_fwd_packed")


def sqa_attn_bwd_workspace_size(B, N, H_q, H_kv, d_head) -> int:
    return int(library().sqa_attn_bwd_workspace_size(B, N, H_q, H_kv, d_head))


def sqa_attn_bwd(q, k, v, out, o_dtype, dout, lse, dq, dk, dv, grad_dtype, B, N, H_q, H_kv,
                 d_head, causal, scale, workspace, workspace_bytes, stream=None) -> None:
    _check(library().sqa_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), int(o_dtype), _ptr(dout),
                             _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), int(grad_dtype),
                             B, N, H_q, H_kv, d_head, int(bool(causal)), float(scale),
                             _ptr(workspace), int(workspace_bytes), _stream(stream)),
           "sqa_attn_bwd")


def sqa_attn_bwd_cross(q, k, v, out, o_dtype, dout, lse, dq, dk, dv, grad_dtype, B, N_q, N_kv, H_q,
                       H_kv, d_head, scale, workspace, workspace_bytes, stream=None) -> None:
    """Gradient of sqa_attn_fwd_cross; workspace sized for N_q query rows."""
    _check(library().sqa_attn_bwd_cross(_ptr(q), _ptr(k), _ptr(v), _ptr(out), int(o_dtype), _ptr(dout),
                                        _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), int(grad_dtype),
                                        B, N_q, N_kv, H_q, H_kv, d_head, float(scale),
                                        _ptr(workspace), int(workspace_bytes), _stream(stream)),
           "sqa_attn_bwd_cross")


def sqa_attn_bwd_window(q, k, v, out, o_dtype, dout, lse, dq, dk, dv, grad_dtype, B, N, H_q, H_kv, d_head,
                        window_left, window_right, scale, workspace, workspace_bytes, stream=None) -> None:
    """Gradient of sqa_attn_fwd_window (same window)."""
    _check(library().sqa_attn_bwd_window(_ptr(q), _ptr(k), _ptr(v), _ptr(out), int(o_dtype), _ptr(dout),
                                         _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), int(grad_dtype),
                                         B, N, H_q, H_kv, d_head, int(window_left), int(window_right),
                                         float(scale), _ptr(workspace), int(workspace_bytes), _stream(stream)),
           "sqa_attn_bwd_window")


def sqa_attn_bwd_packed(qkv, out, o_dtype, dout, lse, dqkv, grad_dtype, B, N, H_q, H_kv, d_head, causal,
                        scale, workspace, workspace_bytes, stream=None) -> None:
    """Gradient of sqa_attn_fwd_packed into a packed dQKV buffer."""
    _check(library().sqa_attn_bwd_packed(_ptr(qkv), _ptr(out), int(o_dtype), _ptr(dout), _ptr(lse), _ptr(dqkv),
                                         int(grad_dtype), B, N, H_q, H_kv, d_head, int(bool(causal)),
                                         float(scale), _ptr(workspace), int(workspace_bytes), _stream(stream)),
           "sqa_attn_bwd_packed")


def sqa_attn_bwd_static(q, k, v, out, o_dtype, dout, lse, dq, dk, dv, grad_dtype, B, N, H_q, H_kv,
                        d_head, causal, scale, stream=None) -> None:
    """sqa_attn_bwd with the library's fixed device scratch instead of a
    caller workspace, for callers that cannot allocate device memory; see
    include/sqa.h for its size limit and sharing rules."""
    _check(library().sqa_attn_bwd_static(_ptr(q), _ptr(k), _ptr(v), _ptr(out), int(o_dtype), _ptr(dout),
                                    _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), int(grad_dtype),
                                    B, N, H_q, H_kv, d_head, int(bool(causal)), float(scale),
                                    _stream(stream)), "sqa_attn_bwd_static")


def sqa_proj(x, w, bias, y, y_dtype, M, K, Nout, stream=None) -> None:
    _check(library().sqa_proj(_ptr(x), _ptr(w), _ptr(bias), _ptr(y), int(y_dtype), M, K, Nout,
                         _stream(stream)), "sqa_proj")


def sqa_gemm(a, a_layout, b, b_layout, bias, c, c_dtype, accumulate, M, N, K, stream=None) -> None:
    _check(library().sqa_gemm(_ptr(a), int(a_layout), _ptr(b), int(b_layout), _ptr(bias), _ptr(c), int(c_dtype),
                              int(bool(accumulate)), M, N, K, _stream(stream)), "sqa_gemm")


def sqa_device_status(stream=None) -> None:
    _check(library().sqa_device_status(_stream(stream)), "sqa_device_status")


def sqa_selftest_wait_timeout(timeout_ms, stream=None) -> None:
    _check(library().sqa_selftest_wait_timeout(int(timeout_ms), _stream(stream)), "sqa_selftest_wait_timeout")
