"""The polynomial 2^x the softmax kernels use for part of their exponentials
(CPU checks).  The coefficients in csrc/sqa_ptx.cuh must be the Remez fit the
fit script derives, and the reduction + polynomial, emulated step by step in
fp32, must stay within 1e-4 relative of 2^x over the range the softmax feeds
it (scaled score minus running max: [-120, 8])."""

import os
import re

import numpy as np

from sparse_query_attention_b200.fit_exp2_poly import remez_exp2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PTX = os.path.join(ROOT, "sparse_query_attention_b200", "csrc", "sqa_ptx.cuh")


def _kernel_coefficients():
    text = open(PTX).read()
    return [float(re.search(rf"kExp2C{i} = ([0-9.e+-]+)f;", text).group(1)) for i in range(4)]


def test_coefficients_are_the_remez_fit():
    fit, err = remez_exp2()
    assert err < 8e-5
    np.testing.assert_allclose(_kernel_coefficients(), fit, rtol=1e-12, atol=1e-15)


def _f32(x):
    return np.float32(x)


def _emulate(x):
    """The device steps in fp32 (fma emulated in fp64 then rounded once)."""
    c0, c1, c2, c3 = (np.float32(c) for c in _kernel_coefficients())
    shift = np.float32(12582912.0)
    x = np.maximum(x.astype(np.float32), np.float32(-120.0))
    t = (x + shift).astype(np.float32)
    n = (t - shift).astype(np.float32)
    f = (x.astype(np.float64) - n.astype(np.float64)).astype(np.float32)
    p = (c3.astype(np.float64) * f + c2).astype(np.float32)
    p = (p.astype(np.float64) * f + c1).astype(np.float32)
    p = (p.astype(np.float64) * f + c0).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def test_emulated_device_steps_match_exp2():
    x = np.concatenate([np.linspace(-120, 8, 400001, dtype=np.float32),
                        np.array([0.0, -0.5, 0.5, -1.5, 1.5, -119.5, 7.999], dtype=np.float32)])
    y = _emulate(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(y - want) / want
    assert rel.max() < 1e-4, rel.max()
