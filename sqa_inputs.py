"""Seeded synthetic inputs for the Sparse Query Attention core and layer.

This module only draws random numbers.  It holds none of the attention
arithmetic, so both the CUDA path and the CPU oracle can consume the same
bf16 bit patterns without sharing any computation.

Recipe (the same for every workload):

* ``torch.Generator`` on the requested device, seeded with ``seed``.
* Tensors are drawn in a fixed order as fp32 N(0, 1) and rounded to bf16
  (round-to-nearest-even, torch's ``.to(torch.bfloat16)``).
  - attention core: Q, K, V, then dO when a gradient is wanted;
  - layer: x, Wq, Wk, Wv, Wo, weights scaled by 0.02 before the rounding.
* Sampled query rows are distinct token indices drawn without replacement by
  ``numpy.random.default_rng(seed)`` and returned sorted.

The CPU and CUDA generators give different streams for the same seed; a test
or benchmark picks one device, draws there, and hands the very same bits to
both sides (copying to the host for the oracle).
"""

from __future__ import annotations

import numpy as np
import torch


def _draw(gen: torch.Generator, shape, std: float, device) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, dtype=torch.float32, device=device)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def attention_inputs(B: int, N: int, H_q: int, H_kv: int, d_head: int, seed: int,
                     with_dout: bool = False, device="cpu") -> dict:
    """Q [B,N,H_q,d], K and V [B,N,H_kv,d] (and dO [B,N,H_q,d]) as bf16."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    out = {
        "q": _draw(gen, (B, N, H_q, d_head), 1.0, device),
        "k": _draw(gen, (B, N, H_kv, d_head), 1.0, device),
        "v": _draw(gen, (B, N, H_kv, d_head), 1.0, device),
    }
    if with_dout:
        out["do"] = _draw(gen, (B, N, H_q, d_head), 1.0, device)
    return out


def cross_attention_inputs(B: int, N_q: int, N_kv: int, H_q: int, H_kv: int, d_head: int, seed: int,
                           with_dout: bool = False, device="cpu") -> dict:
    """Cross / memory attention: Q (and dO) [B,N_q,H_q,d], K and V
    [B,N_kv,H_kv,d], bf16, drawn in the same order as attention_inputs."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    out = {
        "q": _draw(gen, (B, N_q, H_q, d_head), 1.0, device),
        "k": _draw(gen, (B, N_kv, H_kv, d_head), 1.0, device),
        "v": _draw(gen, (B, N_kv, H_kv, d_head), 1.0, device),
    }
    if with_dout:
        out["do"] = _draw(gen, (B, N_q, H_q, d_head), 1.0, device)
    return out


def layer_inputs(B: int, N: int, d_model: int, H_q: int, H_kv: int, d_head: int,
                 seed: int, device="cpu") -> dict:
    """x [B*N, d_model]; Wq [H_q*d, d_model]; Wk, Wv [H_kv*d, d_model];
    Wo [d_model, H_q*d]; all bf16, weights with standard deviation 0.02."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    return {
        "x": _draw(gen, (B * N, d_model), 1.0, device),
        "wq": _draw(gen, (H_q * d_head, d_model), 0.02, device),
        "wk": _draw(gen, (H_kv * d_head, d_model), 0.02, device),
        "wv": _draw(gen, (H_kv * d_head, d_model), 0.02, device),
        "wo": _draw(gen, (d_model, H_q * d_head), 0.02, device),
    }


def sample_rows(N: int, count: int, seed: int) -> np.ndarray:
    """``count`` distinct token indices in [0, N), sorted."""
    rng = np.random.default_rng(int(seed))
    count = min(int(count), int(N))
    return np.sort(rng.choice(N, size=count, replace=False)).astype(np.int64)
