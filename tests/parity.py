"""Shared helpers for the GPU parity tests: the tolerance and the calls that
run the CUDA path through the C ABI on seeded inputs.

Every comparison is recorded in RECORDS (what was compared, max |err|,
relative L2 error, max |ref|, the bound that was applied, and the
elementwise allclose reading with its worst element); tests/conftest.py
prints them at the end of the run and writes them as JSON to the path in
$SQA_PARITY_REPORT when that is set.
"""

from __future__ import annotations

import math
import os

import numpy as np
import torch

# bf16 inputs, fp32 accumulation: max |err| <= 2e-2 and relative L2 error
# <= 1e-2, per output tensor.
ATOL = 2e-2
RTOL_L2 = 1e-2
# The elementwise reading of the same tolerance, |g - o| <= 2e-2 + 1e-2 |o|
# for every element: reported for every comparison, not asserted.
ELEM_ATOL = 2e-2
ELEM_RTOL = 1e-2

RECORDS: list[dict] = []


def errors(got, want):
    """max |got - want| and ||got - want|| / ||want||.  An exactly zero
    reference (the dQ and dK of a window with one visible key per row, where
    the softmax Jacobian of a single key vanishes) has no relative error: it
    is reported as 0, and only the absolute bound applies."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    diff = got - want
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    norm = float(np.linalg.norm(want.ravel()))
    rel_l2 = float(np.linalg.norm(diff.ravel()) / norm) if norm > 0 else 0.0
    return max_abs, rel_l2


def elementwise(got, want):
    """The elementwise allclose reading: whether every element satisfies
    |g - o| <= ELEM_ATOL + ELEM_RTOL |o|, the fraction that does not, and the
    element furthest beyond its allowance."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    if got.size == 0:
        return {"allclose": True, "frac_outside": 0.0, "worst": None}
    err = np.abs(got - want)
    allowed = ELEM_ATOL + ELEM_RTOL * np.abs(want)
    excess = err - allowed
    i = int(np.argmax(excess))
    idx = [int(v) for v in np.unravel_index(i, got.shape)]
    return {"allclose": bool((excess <= 0).all()), "frac_outside": float((excess > 0).mean()),
            "worst": {"index": idx, "got": float(got.flat[i]), "want": float(want.flat[i]),
                      "abs_err": float(err.flat[i]), "allowed": float(allowed.flat[i])}}


def _record(what, got, want, max_abs, rel_l2, bound, passed):
    want = np.asarray(want, dtype=np.float64)
    max_ref = float(np.abs(want).max()) if want.size else 0.0
    RECORDS.append({
        "test": os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0],
        "what": what, "shape": list(np.shape(want)),
        "max_abs": max_abs, "rel_l2": rel_l2, "max_ref": max_ref,
        "max_abs_over_max_ref": max_abs / max_ref if max_ref > 0 else 0.0,
        "bound": bound, "pass": bool(passed), **elementwise(got, want)})


def assert_close(got, want, what=""):
    got = np.asarray(got, dtype=np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    max_abs, rel_l2 = errors(got, want)
    ok = max_abs <= ATOL and rel_l2 <= RTOL_L2
    _record(what, got, want, max_abs, rel_l2, f"max|err|<={ATOL:g}", ok)
    assert ok, f"{what}: max|err|={max_abs:.3e} relL2={rel_l2:.3e}"
    return max_abs, rel_l2


def assert_close_scaled(got, want, what=""):
    """The same bounds relative to the tensor's scale, for outputs whose
    entries are far from unit size (the layer's weight gradients sum over
    B*N tokens and reach ~10; dK/dV summed over up to 128 query heads reach
    ~20): the bf16 rounding of the intermediate or output gradients (~2^-9
    relative per element) then shows up as an absolute error proportional to
    |ref|, while the relative L2 error stays ~2e-3.
    Pass iff max|err| <= 2e-2 * max(1, max|ref|) and relL2 <= 1e-2.  The
    record keeps max|err| itself, so how far past 2e-2 the tensor went is in
    the report."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    max_abs, rel_l2 = errors(got, want)
    scale = max(1.0, float(np.abs(want).max()))
    ok = max_abs <= ATOL * scale and rel_l2 <= RTOL_L2
    _record(what, got, want, max_abs, rel_l2, f"max|err|<={ATOL:g}*{scale:.3g}", ok)
    assert ok, f"{what}: max|err|={max_abs:.3e} (scale {scale:.2f}) relL2={rel_l2:.3e}"
    return max_abs, rel_l2


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def run_fwd(sqa, q, k, v, causal, scale=None, out_dtype=torch.float32, with_lse=True):
    """Runs sqa_attn_fwd_ex on device tensors; returns (o [B,N,H_q,d], lse)."""
    B, N, H_q, d = q.shape
    H_kv = k.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    out = torch.empty((B, N, H_q, d), dtype=out_dtype, device=q.device)
    lse = torch.empty((B, H_q, N), dtype=torch.float32, device=q.device) if with_lse else None
    dt = sqa.SQA_DT_BF16 if out_dtype == torch.bfloat16 else sqa.SQA_DT_F32
    sqa.sqa_attn_fwd_ex(q, k, v, out, dt, lse, B, N, H_q, H_kv, d, causal, scale)
    return out, lse


def run_bwd(sqa, q, k, v, o, do, lse, causal, scale=None, grad_dtype=torch.float32):
    B, N, H_q, d = q.shape
    H_kv = k.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dq = torch.empty_like(q, dtype=grad_dtype)
    dk = torch.empty_like(k, dtype=grad_dtype)
    dv = torch.empty_like(v, dtype=grad_dtype)
    wsb = sqa.sqa_attn_bwd_workspace_size(B, N, H_q, H_kv, d)
    ws = torch.empty(wsb, dtype=torch.uint8, device=q.device)
    od = sqa.SQA_DT_BF16 if o.dtype == torch.bfloat16 else sqa.SQA_DT_F32
    gd = sqa.SQA_DT_BF16 if grad_dtype == torch.bfloat16 else sqa.SQA_DT_F32
    sqa.sqa_attn_bwd(q, k, v, o, od, do, lse, dq, dk, dv, gd, B, N, H_q, H_kv, d, causal, scale, ws, wsb)
    return dq, dk, dv
