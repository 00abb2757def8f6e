"""Pins for the fp64 oracle, independent of the oracle's own code (CPU only).

Each check ties the oracle to something other than itself: hand-derived
closed forms (tests/golden), a pure-Python brute force with a different
evaluation order (unstabilised softmax, math.fsum), a library routine
(torch scaled_dot_product_attention and autograd in fp64), finite
differences, invariants of softmax attention, and the closed-form FLOP count
behind the query-head reduction ("Sparse Query Attention (SQA): A
Computationally Efficient Attention Mechanism with Query Heads Reduction",
abstract: attention FLOPs fall in proportion to the number of query heads).
"""

import itertools
import json
import math
import os
import re

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import (attention_backward, attention_decode, attention_forward, projection, projection_backward,
                    sqa_layer_backward, sqa_layer_forward)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_form_cases.json")


# ----------------------------------------------------------------------------
# Independent brute force: nested Python loops, unstabilised softmax, fsum.
# It also counts the multiply-adds of the two contractions it performs.
# ----------------------------------------------------------------------------
class _Counter:
    def __init__(self):
        self.qk = 0
        self.pv = 0


def brute_attention(q, k, v, causal, scale, counter=None):
    B, N, H_q, d = q.shape
    H_kv = k.shape[2]
    G = H_q // H_kv
    o = np.zeros((B, N, H_q, d))
    lse = np.zeros((B, H_q, N))
    for b in range(B):
        for h in range(H_q):
            j = h // G
            for t in range(N):
                keys = range(t + 1) if causal else range(N)
                e = []
                for u in keys:
                    s = scale * math.fsum(float(q[b, t, h, c]) * float(k[b, u, j, c]) for c in range(d))
                    if counter is not None:
                        counter.qk += d
                    e.append(math.exp(s))
                z = math.fsum(e)
                for c in range(d):
                    o[b, t, h, c] = math.fsum(e[i] * float(v[b, u, j, c]) for i, u in enumerate(keys)) / z
                    if counter is not None:
                        counter.pv += len(e)
                lse[b, h, t] = math.log(z)
    return o, lse


def _rand(shape, rng, scale=1.0):
    return rng.standard_normal(shape) * scale


def _expand(x):
    """Numbers, or the fixture's small expressions in ln3 / ln4."""
    if isinstance(x, str):
        expr = re.sub(r"(\d)(ln[34])", r"\1*\2", x)
        return float(eval(expr, {"__builtins__": {}}, {"ln3": math.log(3.0), "ln4": math.log(4.0)}))
    return float(x)


def _arr(nested):
    def walk(x):
        return [walk(y) for y in x] if isinstance(x, list) else _expand(x)
    return np.array(walk(nested), dtype=np.float64)


# ----------------------------------------------------------------------------
# Closed forms worked by hand
# ----------------------------------------------------------------------------
def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_closed_form_cases(case):
    q = _arr(case["q"])[None]
    k = _arr(case["k"])[None]
    v = _arr(case["v"])[None]
    o, lse = attention_forward(q, k, v, case["causal"], case["scale"])
    np.testing.assert_allclose(o[0], _arr(case["o"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0], _arr(case["lse"]), rtol=1e-15, atol=1e-12)
    if "dq" in case:
        dq, dk, dv = attention_backward(q, k, v, _arr(case["do"])[None], case["causal"], case["scale"])
        np.testing.assert_allclose(dq[0], _arr(case["dq"]), atol=1e-12)
        np.testing.assert_allclose(dk[0], _arr(case["dk"]), atol=1e-12)
        np.testing.assert_allclose(dv[0], _arr(case["dv"]), atol=1e-12)


def test_golden_expander():
    assert _expand("-1.5ln3") == pytest.approx(-1.5 * math.log(3))
    assert _expand("1+ln3/1000") == pytest.approx(1 + math.log(3) / 1000)
    assert _expand("1000+ln4") == pytest.approx(1000 + math.log(4))


# ----------------------------------------------------------------------------
# Brute force on tiny inputs
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("heads", [(1, 1), (2, 1), (2, 2), (4, 2), (4, 1)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(1, 1), (3, 2), (6, 4)])
def test_brute_force_tiny(heads, causal, N, d):
    H_q, H_kv = heads
    rng = np.random.default_rng(N * 100 + d * 10 + H_q + causal)
    B = 2
    q = _rand((B, N, H_q, d), rng)
    k = _rand((B, N, H_kv, d), rng)
    v = _rand((B, N, H_kv, d), rng)
    scale = 1.0 / math.sqrt(d)
    o, lse = attention_forward(q, k, v, causal, scale)
    ob, lseb = brute_attention(q, k, v, causal, scale)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lseb, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------
# Reduction to standard attention: torch SDPA (fp64, CPU) as a library check
# ----------------------------------------------------------------------------
def _sdpa(q, k, v, causal, scale, gqa):
    tq = torch.from_numpy(q).permute(0, 2, 1, 3)
    tk = torch.from_numpy(k).permute(0, 2, 1, 3)
    tv = torch.from_numpy(v).permute(0, 2, 1, 3)
    o = F.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale, enable_gqa=gqa)
    return o.permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("heads", [(4, 4), (8, 4), (8, 2), (4, 1), (16, 4)])
@pytest.mark.parametrize("causal", [False, True])
def test_matches_sdpa(heads, causal):
    H_q, H_kv = heads
    rng = np.random.default_rng(7 + H_q * 3 + H_kv + causal)
    B, N, d = 2, 37, 16
    q, k, v = _rand((B, N, H_q, d), rng), _rand((B, N, H_kv, d), rng), _rand((B, N, H_kv, d), rng)
    scale = 1.0 / math.sqrt(d)
    o, _ = attention_forward(q, k, v, causal, scale)
    np.testing.assert_allclose(o, _sdpa(q, k, v, causal, scale, H_q != H_kv), rtol=0, atol=1e-12)


def test_gqa_expansion_identity():
    """SQA(H_q, H_kv) equals MHA with H_q heads on K/V repeated G times
    (contiguous groups); gradients of K/V are the group sums of the MHA ones."""
    rng = np.random.default_rng(11)
    B, N, H_q, H_kv, d = 2, 19, 8, 2, 8
    G = H_q // H_kv
    q, k, v = _rand((B, N, H_q, d), rng), _rand((B, N, H_kv, d), rng), _rand((B, N, H_kv, d), rng)
    do = _rand((B, N, H_q, d), rng)
    kr, vr = np.repeat(k, G, axis=2), np.repeat(v, G, axis=2)
    for causal in (False, True):
        o, lse = attention_forward(q, k, v, causal, 0.3)
        o2, lse2 = attention_forward(q, kr, vr, causal, 0.3)
        np.testing.assert_allclose(o, o2, atol=1e-13)
        np.testing.assert_allclose(lse, lse2, atol=1e-13)
        dq, dk, dv = attention_backward(q, k, v, do, causal, 0.3)
        dq2, dk2, dv2 = attention_backward(q, kr, vr, do, causal, 0.3)
        np.testing.assert_allclose(dq, dq2, atol=1e-12)
        np.testing.assert_allclose(dk, dk2.reshape(B, N, H_kv, G, d).sum(3), atol=1e-12)
        np.testing.assert_allclose(dv, dv2.reshape(B, N, H_kv, G, d).sum(3), atol=1e-12)


# ----------------------------------------------------------------------------
# Softmax and attention invariants
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_rows_sum_to_one_and_mask_is_zero(causal):
    """With d = N and V the identity (v[u] = e_u), o[t] is the probability
    row itself: it sums to 1, and masked entries are exactly 0."""
    rng = np.random.default_rng(3)
    B, N, H_q, H_kv = 1, 12, 4, 2
    q = _rand((B, N, H_q, N), rng)
    k = _rand((B, N, H_kv, N), rng)
    v = np.broadcast_to(np.eye(N)[None, :, None, :], (B, N, H_kv, N)).copy()
    o, _ = attention_forward(q, k, v, causal, 0.5)
    np.testing.assert_allclose(o.sum(axis=-1), 1.0, atol=1e-12)
    assert (o >= 0).all()
    if causal:
        upper = np.triu(np.ones((N, N), dtype=bool), 1)
        assert (o[0][:, 0][upper] == 0).all()
        assert (o[0].transpose(1, 0, 2)[:, upper] == 0).all()


@pytest.mark.parametrize("causal", [False, True])
def test_identical_keys_give_mean_of_v(causal):
    rng = np.random.default_rng(5)
    B, N, H_q, H_kv, d = 2, 9, 4, 2, 3
    q = _rand((B, N, H_q, d), rng)
    k = np.broadcast_to(_rand((B, 1, H_kv, d), rng), (B, N, H_kv, d)).copy()
    v = _rand((B, N, H_kv, d), rng)
    do = _rand((B, N, H_q, d), rng)
    o, _ = attention_forward(q, k, v, causal, 0.7)
    G = H_q // H_kv
    for t in range(N):
        keys = slice(0, t + 1) if causal else slice(0, N)
        for h in range(H_q):
            np.testing.assert_allclose(o[:, t, h], v[:, keys, h // G].mean(axis=1), atol=1e-13)
    dq, _, _ = attention_backward(q, k, v, do, causal, 0.7)
    np.testing.assert_allclose(dq, 0.0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_invariants(causal):
    """sum_u dS_tu = 0 gives sum_u dk[u] = 0 per kv head; and
    sum_u dv[u, j] = sum over the group's heads and all t of do."""
    rng = np.random.default_rng(8)
    B, N, H_q, H_kv, d = 2, 14, 6, 2, 5
    q, k, v = _rand((B, N, H_q, d), rng), _rand((B, N, H_kv, d), rng), _rand((B, N, H_kv, d), rng)
    do = _rand((B, N, H_q, d), rng)
    dq, dk, dv = attention_backward(q, k, v, do, causal, 0.4)
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)
    G = H_q // H_kv
    want = do.reshape(B, N, H_kv, G, d).sum(axis=(1, 3))
    np.testing.assert_allclose(dv.sum(axis=1), want, atol=1e-12)


# ----------------------------------------------------------------------------
# Gradients: central differences of the brute force, and torch autograd
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_backward_finite_differences(causal):
    rng = np.random.default_rng(21 + causal)
    B, N, H_q, H_kv, d = 1, 4, 2, 1, 3
    q, k, v = _rand((B, N, H_q, d), rng), _rand((B, N, H_kv, d), rng), _rand((B, N, H_kv, d), rng)
    do = _rand((B, N, H_q, d), rng)
    scale = 0.6
    dq, dk, dv = attention_backward(q, k, v, do, causal, scale)
    eps = 1e-6

    def loss(q_, k_, v_):
        o, _ = brute_attention(q_, k_, v_, causal, scale)
        return math.fsum((o * do).ravel())

    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        for idx in itertools.product(*[range(n) for n in x.shape]):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": q, "k": k, "v": v}
            args_m = {"q": q, "k": k, "v": v}
            args_p[name], args_m[name] = xp, xm
            fd[idx] = (loss(**{a + "_": b for a, b in args_p.items()})
                       - loss(**{a + "_": b for a, b in args_m.items()})) / (2 * eps)
        err = np.abs(fd - g).max() / max(np.abs(g).max(), 1e-300)
        assert err < 1e-6, (name, err)


@pytest.mark.parametrize("heads", [(4, 4), (8, 4), (4, 1)])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_autograd(heads, causal):
    H_q, H_kv = heads
    rng = np.random.default_rng(31 + H_q + H_kv + causal)
    B, N, d = 2, 23, 8
    q, k, v = _rand((B, N, H_q, d), rng), _rand((B, N, H_kv, d), rng), _rand((B, N, H_kv, d), rng)
    do = _rand((B, N, H_q, d), rng)
    scale = 1 / math.sqrt(d)
    tq, tk, tv = (torch.from_numpy(a.copy()).permute(0, 2, 1, 3).requires_grad_() for a in (q, k, v))
    o = F.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale, enable_gqa=H_q != H_kv)
    o.backward(torch.from_numpy(do).permute(0, 2, 1, 3))
    dq, dk, dv = attention_backward(q, k, v, do, causal, scale)
    np.testing.assert_allclose(dq, tq.grad.permute(0, 2, 1, 3).numpy(), atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.permute(0, 2, 1, 3).numpy(), atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.permute(0, 2, 1, 3).numpy(), atol=1e-12)


# ----------------------------------------------------------------------------
# Sampled rows, chunk boundaries
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_sampled_rows_equal_full_rows(causal):
    rng = np.random.default_rng(13)
    B, N, H_q, H_kv, d = 1, 600, 4, 2, 8   # N spans several 256-row chunks
    q, k, v = _rand((B, N, H_q, d), rng), _rand((B, N, H_kv, d), rng), _rand((B, N, H_kv, d), rng)
    o, lse = attention_forward(q, k, v, causal, 0.35)
    rows = np.array([0, 1, 255, 256, 257, 511, 512, 599])
    os_, lses = attention_forward(q, k, v, causal, 0.35, rows=rows)
    np.testing.assert_allclose(os_, o[:, rows], atol=1e-13)
    np.testing.assert_allclose(lses, lse[:, :, rows], atol=1e-13)
    ob, lseb = brute_attention(q[:, :40], k[:, :40], v[:, :40], causal, 0.35) if causal else (None, None)
    if causal:  # causal rows < 40 only see the first 40 keys
        np.testing.assert_allclose(o[:, :40], ob, atol=1e-12)
        np.testing.assert_allclose(lse[:, :, :40], lseb, atol=1e-12)


# ----------------------------------------------------------------------------
# FLOP accounting: the query-head reduction factor
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [False, True])
def test_flop_count_scales_with_query_heads(causal):
    """The brute force's counted multiply-adds per contraction equal
    B * H_q * P_c * d (P_c = N(N+1)/2 causal, N^2 otherwise), so MHA / SQA
    costs H / H_q exactly, independent of H_kv."""
    B, N, d, H = 1, 7, 2, 8
    counts = {}
    for H_q, H_kv in ((8, 8), (8, 2), (4, 4), (4, 1), (2, 2)):
        rng = np.random.default_rng(0)
        c = _Counter()
        brute_attention(_rand((B, N, H_q, d), rng), _rand((B, N, H_kv, d), rng),
                        _rand((B, N, H_kv, d), rng), causal, 1.0, counter=c)
        P_c = N * (N + 1) // 2 if causal else N * N
        assert c.qk == B * H_q * P_c * d
        assert c.pv == B * H_q * P_c * d
        counts[(H_q, H_kv)] = c.qk + c.pv
    assert counts[(8, 8)] == counts[(8, 2)]
    for (H_q, H_kv), n in counts.items():
        assert counts[(H, H)] * H_q == n * H


# ----------------------------------------------------------------------------
# Projections and the layer
# ----------------------------------------------------------------------------
def test_projection_naive_loop_and_matmul():
    rng = np.random.default_rng(17)
    M, K, Nout = 5, 7, 3
    x, w, bias = _rand((M, K), rng), _rand((Nout, K), rng), _rand((Nout,), rng)
    y = projection(x, w, bias)
    for m in range(M):
        for n in range(Nout):
            assert y[m, n] == pytest.approx(math.fsum(x[m, c] * w[n, c] for c in range(K)) + bias[n], abs=1e-13)
    big_x, big_w = _rand((64, 48), rng), _rand((40, 48), rng)
    ref = torch.from_numpy(big_x) @ torch.from_numpy(big_w).T
    np.testing.assert_allclose(projection(big_x, big_w), ref.numpy(), atol=1e-12)


def test_layer_against_torch_composition():
    """The layer equals nn.functional.linear -> SDPA (GQA) -> linear in fp64."""
    rng = np.random.default_rng(19)
    B, N, d_model, H_q, H_kv, dh = 2, 17, 32, 4, 2, 8
    x = _rand((B * N, d_model), rng)
    wq, wk, wv = _rand((H_q * dh, d_model), rng, .1), _rand((H_kv * dh, d_model), rng, .1), _rand((H_kv * dh, d_model), rng, .1)
    wo = _rand((d_model, H_q * dh), rng, .1)
    out = sqa_layer_forward(x, wq, wk, wv, wo, B, N, H_q, H_kv, dh, causal=True)
    tx = torch.from_numpy(x)
    tq = F.linear(tx, torch.from_numpy(wq)).view(B, N, H_q, dh).transpose(1, 2)
    tk = F.linear(tx, torch.from_numpy(wk)).view(B, N, H_kv, dh).transpose(1, 2)
    tv = F.linear(tx, torch.from_numpy(wv)).view(B, N, H_kv, dh).transpose(1, 2)
    to = F.scaled_dot_product_attention(tq, tk, tv, is_causal=True, enable_gqa=True)
    ty = F.linear(to.transpose(1, 2).reshape(B * N, H_q * dh), torch.from_numpy(wo))
    np.testing.assert_allclose(out["y"], ty.numpy(), atol=1e-12)


def test_projection_backward_brute_force():
    """dx = dy w and dw = dy^T x against explicit sums (tiny)."""
    rng = np.random.default_rng(23)
    M, K, Nout = 4, 3, 5
    x, w, dy = _rand((M, K), rng), _rand((Nout, K), rng), _rand((M, Nout), rng)
    dx, dw = projection_backward(x, w, dy)
    for m in range(M):
        for k in range(K):
            assert dx[m, k] == pytest.approx(math.fsum(dy[m, n] * w[n, k] for n in range(Nout)), abs=1e-13)
    for n in range(Nout):
        for k in range(K):
            assert dw[n, k] == pytest.approx(math.fsum(dy[m, n] * x[m, k] for m in range(M)), abs=1e-13)


@pytest.mark.parametrize("heads", [(4, 2), (4, 4), (4, 1)])
def test_layer_backward_matches_autograd(heads):
    """Every layer gradient equals torch autograd (fp64) through
    linear -> SDPA (GQA) -> linear."""
    H_q, H_kv = heads
    rng = np.random.default_rng(29 + H_q + H_kv)
    B, N, d_model, dh = 2, 13, 16, 8
    x = _rand((B * N, d_model), rng)
    wq = _rand((H_q * dh, d_model), rng, .2)
    wk, wv = _rand((H_kv * dh, d_model), rng, .2), _rand((H_kv * dh, d_model), rng, .2)
    wo = _rand((d_model, H_q * dh), rng, .2)
    dy = _rand((B * N, d_model), rng)
    g = sqa_layer_backward(x, wq, wk, wv, wo, dy, B, N, H_q, H_kv, dh, causal=True)
    t = {n: torch.from_numpy(a.copy()).requires_grad_() for n, a in
         (("x", x), ("wq", wq), ("wk", wk), ("wv", wv), ("wo", wo))}
    tq = F.linear(t["x"], t["wq"]).view(B, N, H_q, dh).transpose(1, 2)
    tk = F.linear(t["x"], t["wk"]).view(B, N, H_kv, dh).transpose(1, 2)
    tv = F.linear(t["x"], t["wv"]).view(B, N, H_kv, dh).transpose(1, 2)
    to = F.scaled_dot_product_attention(tq, tk, tv, is_causal=True, enable_gqa=H_q != H_kv)
    ty = F.linear(to.transpose(1, 2).reshape(B * N, H_q * dh), t["wo"])
    ty.backward(torch.from_numpy(dy))
    np.testing.assert_allclose(g["dx"], t["x"].grad.numpy(), atol=1e-12)
    for n in ("wq", "wk", "wv", "wo"):
        np.testing.assert_allclose(g["d" + n], t[n].grad.numpy(), atol=1e-12)


@pytest.mark.parametrize("N_q,N_kv,heads", [(7, 19, (4, 2)), (33, 5, (4, 4)), (16, 64, (8, 1))])
def test_cross_attention_matches_sdpa_and_autograd(N_q, N_kv, heads):
    """Queries and keys of different lengths (memory attention): output and
    all three gradients equal torch SDPA / autograd in fp64."""
    H_q, H_kv = heads
    rng = np.random.default_rng(N_q * 7 + N_kv)
    B, d = 2, 8
    q, k, v = _rand((B, N_q, H_q, d), rng), _rand((B, N_kv, H_kv, d), rng), _rand((B, N_kv, H_kv, d), rng)
    do = _rand((B, N_q, H_q, d), rng)
    scale = 1 / math.sqrt(d)
    o, lse = attention_forward(q, k, v, False, scale)
    tq, tk, tv = (torch.from_numpy(a.copy()).permute(0, 2, 1, 3).requires_grad_() for a in (q, k, v))
    to = F.scaled_dot_product_attention(tq, tk, tv, scale=scale, enable_gqa=H_q != H_kv)
    np.testing.assert_allclose(o, to.detach().permute(0, 2, 1, 3).numpy(), atol=1e-12)
    ob, lseb = brute_attention_cross(q, k, v, scale)
    np.testing.assert_allclose(lse, lseb, atol=1e-12)
    to.backward(torch.from_numpy(do).permute(0, 2, 1, 3))
    dq, dk, dv = attention_backward(q, k, v, do, False, scale)
    np.testing.assert_allclose(dq, tq.grad.permute(0, 2, 1, 3).numpy(), atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.permute(0, 2, 1, 3).numpy(), atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.permute(0, 2, 1, 3).numpy(), atol=1e-12)


def brute_attention_cross(q, k, v, scale):
    """Non-causal brute force for different query / key lengths (fsum)."""
    B, N_q, H_q, d = q.shape
    N_kv, H_kv = k.shape[1], k.shape[2]
    G = H_q // H_kv
    o = np.zeros(q.shape)
    lse = np.zeros((B, H_q, N_q))
    for b in range(B):
        for h in range(H_q):
            for t in range(N_q):
                e = [math.exp(scale * math.fsum(q[b, t, h, c] * k[b, u, h // G, c] for c in range(d)))
                     for u in range(N_kv)]
                z = math.fsum(e)
                for c in range(d):
                    o[b, t, h, c] = math.fsum(e[u] * v[b, u, h // G, c] for u in range(N_kv)) / z
                lse[b, h, t] = math.log(z)
    return o, lse


def test_causal_cross_attention_is_rejected():
    with pytest.raises(ValueError):
        attention_forward(np.zeros((1, 3, 1, 2)), np.zeros((1, 5, 1, 2)), np.zeros((1, 5, 1, 2)), True, 1.0)


def test_rejects_bad_head_counts():
    q = np.zeros((1, 2, 3, 4))
    k = np.zeros((1, 2, 2, 4))
    with pytest.raises(ValueError):
        attention_forward(q, k, k, False, 1.0)


# ---------------------------------------------------------------------------
# Sliding-window (local) attention
# ---------------------------------------------------------------------------
def brute_attention_window(q, k, v, scale, left, right, causal=False):
    """fsum brute force; the visible keys of query t are listed explicitly:
    max(0, t - left) .. min(N - 1, t + right), capped at t when causal."""
    B, N, H_q, d = q.shape
    G = H_q // k.shape[2]
    o = np.zeros(q.shape)
    lse = np.zeros((B, H_q, N))
    for b in range(B):
        for h in range(H_q):
            for t in range(N):
                last = min(N - 1, t + right)
                if causal:
                    last = min(last, t)
                keys = list(range(max(0, t - left), last + 1))
                e = [math.exp(scale * math.fsum(q[b, t, h, c] * k[b, u, h // G, c] for c in range(d))) for u in keys]
                z = math.fsum(e)
                for c in range(d):
                    o[b, t, h, c] = math.fsum(e[i] * v[b, u, h // G, c] for i, u in enumerate(keys)) / z
                lse[b, h, t] = math.log(z)
    return o, lse


@pytest.mark.parametrize("left,right,causal", [(2, 0, False), (1, 3, False), (0, 0, False), (3, 3, True),
                                               (9, 9, False)])
def test_window_brute_force(left, right, causal):
    rng = np.random.default_rng(left * 10 + right)
    B, N, H_q, H_kv, d = 1, 7, 4, 2, 3
    q, k, v = _rand((B, N, H_q, d), rng), _rand((B, N, H_kv, d), rng), _rand((B, N, H_kv, d), rng)
    o, lse = attention_forward(q, k, v, causal, 0.7, window=(left, right))
    ob, lb = brute_attention_window(q, k, v, 0.7, left, right, causal)
    np.testing.assert_allclose(o, ob, atol=1e-12)
    np.testing.assert_allclose(lse, lb, atol=1e-12)


def _band_mask(N, left, right):
    t = torch.arange(N)[:, None]
    u = torch.arange(N)[None, :]
    return (u >= t - left) & (u <= t + right)


@pytest.mark.parametrize("left,right,heads", [(4, 0, (4, 2)), (2, 5, (4, 4)), (0, 6, (8, 1))])
def test_window_matches_sdpa_mask_and_autograd(left, right, heads):
    """The window as an explicit boolean mask handed to torch SDPA (fp64):
    output, and all three gradients through autograd."""
    H_q, H_kv = heads
    rng = np.random.default_rng(100 + left + 7 * right)
    B, N, d = 2, 13, 8
    q, k, v = _rand((B, N, H_q, d), rng), _rand((B, N, H_kv, d), rng), _rand((B, N, H_kv, d), rng)
    do = _rand((B, N, H_q, d), rng)
    scale = 1 / math.sqrt(d)
    o, _ = attention_forward(q, k, v, False, scale, window=(left, right))
    tq, tk, tv = (torch.from_numpy(a.copy()).permute(0, 2, 1, 3).requires_grad_() for a in (q, k, v))
    to = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=_band_mask(N, left, right), scale=scale,
                                        enable_gqa=H_q != H_kv)
    np.testing.assert_allclose(o, to.detach().permute(0, 2, 1, 3).numpy(), atol=1e-12)
    to.backward(torch.from_numpy(do).permute(0, 2, 1, 3))
    dq, dk, dv = attention_backward(q, k, v, do, False, scale, window=(left, right))
    np.testing.assert_allclose(dq, tq.grad.permute(0, 2, 1, 3).numpy(), atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.permute(0, 2, 1, 3).numpy(), atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.permute(0, 2, 1, 3).numpy(), atol=1e-12)


def test_window_degenerate_cases():
    """(0, 0): each token sees only itself, so O = V of its own token, LSE is
    its own scaled score, and dQ = dK = 0 with dV = the group sum of dO.
    (N, 0) is the causal mask and (N, N) no mask at all."""
    rng = np.random.default_rng(8)
    B, N, H_q, H_kv, d = 2, 9, 4, 2, 5
    q, k, v = _rand((B, N, H_q, d), rng), _rand((B, N, H_kv, d), rng), _rand((B, N, H_kv, d), rng)
    do = _rand((B, N, H_q, d), rng)
    o, lse = attention_forward(q, k, v, False, 0.3, window=(0, 0))
    kx, vx = np.repeat(k, 2, axis=2), np.repeat(v, 2, axis=2)
    np.testing.assert_allclose(o, vx, atol=1e-14)
    np.testing.assert_allclose(lse, 0.3 * np.einsum("bthc,bthc->bht", q, kx), atol=1e-13)
    dq, dk, dv = attention_backward(q, k, v, do, False, 0.3, window=(0, 0))
    np.testing.assert_allclose(dq, 0, atol=1e-14)
    np.testing.assert_allclose(dk, 0, atol=1e-14)
    np.testing.assert_allclose(dv, do.reshape(B, N, H_kv, 2, d).sum(axis=3), atol=1e-14)
    for win, causal in (((N, 0), True), ((N, N), False)):
        ow, lw = attention_forward(q, k, v, False, 0.3, window=win)
        oc, lc = attention_forward(q, k, v, causal, 0.3)
        np.testing.assert_allclose(ow, oc, atol=1e-13)
        np.testing.assert_allclose(lw, lc, atol=1e-13)


def test_window_gradient_invariants():
    """Softmax rows still sum to one inside the window: sum_u dK = 0 per KV
    head and sum_u dV = sum of dO over the group's heads and all tokens."""
    rng = np.random.default_rng(12)
    B, N, H_q, H_kv, d = 1, 11, 6, 2, 4
    q, k, v = _rand((B, N, H_q, d), rng), _rand((B, N, H_kv, d), rng), _rand((B, N, H_kv, d), rng)
    do = _rand((B, N, H_q, d), rng)
    dq, dk, dv = attention_backward(q, k, v, do, False, 0.5, window=(3, 1))
    np.testing.assert_allclose(dk.sum(axis=1), 0, atol=1e-12)
    np.testing.assert_allclose(dv.sum(axis=1), do.reshape(B, N, H_kv, 3, d).sum(axis=(1, 3)), atol=1e-12)


def test_window_rejects_bad_arguments():
    z = np.zeros((1, 4, 1, 2))
    with pytest.raises(ValueError):
        attention_forward(z, z, z, False, 1.0, window=(-1, 0))
    with pytest.raises(ValueError):
        attention_forward(z, np.zeros((1, 5, 1, 2)), np.zeros((1, 5, 1, 2)), False, 1.0, window=(2, 2))


# ---------------------------------------------------------------------------
# KV-cache decode
# ---------------------------------------------------------------------------
def _decode_case(rng, B, n_new, H_q, H_kv, d, lens, L_max):
    q = _rand((B, n_new, H_q, d), rng)
    kc = _rand((B, L_max, H_kv, d), rng)
    vc = _rand((B, L_max, H_kv, d), rng)
    return q, kc, vc, np.asarray(lens)


@pytest.mark.parametrize("n_new,heads", [(1, (4, 2)), (3, (4, 4)), (2, (8, 1))])
def test_decode_matches_sdpa_last_rows(n_new, heads):
    """Decoding n_new tokens equals the last n_new rows of causal attention
    over the sequence's first len_b tokens (torch SDPA, fp64), per sequence,
    with ragged lengths."""
    H_q, H_kv = heads
    rng = np.random.default_rng(40 + n_new)
    B, d, L_max = 3, 8, 23
    lens = [23, 5, 14][:B]
    q, kc, vc, lens = _decode_case(rng, B, n_new, H_q, H_kv, d, lens, L_max)
    scale = 1 / math.sqrt(d)
    o, lse = attention_decode(q, kc, vc, lens, scale)
    for b in range(B):
        L = lens[b]
        qf = _rand((L, H_q, d), rng)      # earlier rows: arbitrary, they only fill the sequence
        qf[L - n_new:] = q[b]
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).permute(1, 0, 2)[None]
        ref = F.scaled_dot_product_attention(t(qf), t(kc[b, :L]), t(vc[b, :L]), is_causal=True, scale=scale,
                                             enable_gqa=H_q != H_kv)
        np.testing.assert_allclose(o[b], ref[0].permute(1, 0, 2).numpy()[L - n_new:], atol=1e-12)


def test_decode_brute_force_and_unused_cache():
    """fsum brute force with explicit key lists; cache entries past len_b
    (here NaN) are never read."""
    rng = np.random.default_rng(5)
    B, n_new, H_q, H_kv, d, L_max = 2, 2, 4, 2, 3, 9
    q, kc, vc, lens = _decode_case(rng, B, n_new, H_q, H_kv, d, [9, 4], L_max)
    kc[1, 4:] = np.nan
    vc[1, 4:] = np.nan
    o, lse = attention_decode(q, kc, vc, lens, 0.6)
    for b in range(B):
        L = int(lens[b])
        for h in range(H_q):
            j = h // 2
            for i in range(n_new):
                keys = range(L - n_new + i + 1)
                e = [math.exp(0.6 * math.fsum(q[b, i, h, c] * kc[b, u, j, c] for c in range(d))) for u in keys]
                z = math.fsum(e)
                for c in range(d):
                    assert abs(o[b, i, h, c] - math.fsum(e[u] * vc[b, u, j, c] for u in keys) / z) < 1e-12
                assert abs(lse[b, h, i] - math.log(z)) < 1e-12


def test_decode_single_key_and_rejects_bad_lengths():
    rng = np.random.default_rng(6)
    q, kc, vc, lens = _decode_case(rng, 1, 1, 2, 1, 4, [1], 5)
    o, lse = attention_decode(q, kc, vc, lens, 0.5)
    np.testing.assert_allclose(o[0, 0], np.repeat(vc[0, 0], 2, axis=0), atol=1e-15)
    np.testing.assert_allclose(lse[0, :, 0], 0.5 * (q[0, 0] @ kc[0, 0, 0]), atol=1e-14)
    for bad in ([0], [6]):
        with pytest.raises(ValueError):
            attention_decode(q, kc, vc, np.asarray(bad), 0.5)
