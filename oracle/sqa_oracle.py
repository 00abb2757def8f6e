"""fp64 CPU oracle for Sparse Query Attention (test infrastructure only).

Imported only by ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py``.  Nothing in the product path imports or calls it.

What it restates, and from where:

* Sparse Query Attention keeps the Grouped Query Attention head sharing but
  cuts the number of *query* heads: H_q < H query heads attend, and each of
  the H_kv key/value heads serves G = H_q / H_kv query heads.
  ("ReactiveAI/GQA-Ref-Micro" model card, introduction;
  "ReactiveAI/xSMQAT-m" model card, introduction;
  "Sparse Query Attention (SQA): A Computationally Efficient Attention
  Mechanism with Query Heads Reduction", abstract.)
* Query and output projections shrink to width H_q * d_head.
  ("ReactiveAI/xSMQAT-m" model card, note on model size;
  "ReactiveAI/GQA-Ref-Micro" model card, note on model size.)
* Causal masking for the decoder models (the training/inference usage on
  both model cards) and no mask for encoder-style work (abstract).
* Sliding-window (local) attention, the spatially sparse pattern SQA is
  set beside ("ReactiveAI/GQA-Ref-Micro" model card, results paragraph: SQA
  as a possible alternative to spatially sparse attention; the paper's
  "Builds on" list includes Longformer): query t sees keys
  t - left <= u <= t + right, optionally together with the causal mask.

The pages print no equations, so the attention itself is the textbook
definition that "extension to Grouped Query Attention" presupposes.  Readings
taken where the pages are silent:

* query head h reads key/value head j = floor(h / G) (contiguous groups);
* scale = 1 / sqrt(d_head), passed explicitly;
* causal: query t sees keys 0..t (diagonal included);
* softmax in natural base, max-subtracted for range only;
* everything in fp64 from inputs given as exact float64 copies of bf16;
  no intermediate rounding anywhere.

Evaluation proceeds one (batch, query head) pair and one chunk of query rows
at a time.  Rows are independent in the definition, so the chunking changes
no arithmetic of any row; it only bounds memory.  Library matmuls (numpy) are
the only primitives used.
"""

from __future__ import annotations

import numpy as np

_CHUNK = 256


def _check_heads(H_q: int, H_kv: int) -> int:
    if H_kv <= 0 or H_q <= 0 or H_q % H_kv != 0:
        raise ValueError(f"H_q={H_q} must be a positive multiple of H_kv={H_kv}")
    return H_q // H_kv


def _check_lengths(N_q: int, N_kv: int, causal: bool) -> None:
    # Cross / memory attention (queries and keys of different lengths) is
    # taken without a mask: "query t sees keys 0..t" has no meaning when the
    # keys are not the same sequence.
    if causal and N_q != N_kv:
        raise ValueError("causal attention needs as many keys as queries")


def _check_window(window, N_q: int, N_kv: int):
    # A window relates query and key positions of one sequence.
    if window is None:
        return None
    left, right = (int(w) for w in window)
    if left < 0 or right < 0:
        raise ValueError("window sides must be >= 0")
    if N_q != N_kv:
        raise ValueError("a window needs as many keys as queries")
    return left, right


def _scores(q_rows, k_head, t_rows, causal, scale, window=None):
    """s[r, u] = scale * <q_r, k_u>, set to -inf where key u is hidden from
    query t_r: u > t_r when causal; u < t_r - left or u > t_r + right for a
    window (left, right).

    Only keys 0..max(t_rows) can be unmasked in the causal case, so the
    columns beyond are never formed; masked entries inside are -inf.
    """
    if causal:
        n_keys = int(t_rows.max()) + 1
        k_head = k_head[:n_keys]
    s = scale * (q_rows @ k_head.T)
    u = np.arange(k_head.shape[0])
    if causal:
        s[u[None, :] > t_rows[:, None]] = -np.inf
    if window is not None:
        left, right = window
        s[u[None, :] < t_rows[:, None] - left] = -np.inf
        s[u[None, :] > t_rows[:, None] + right] = -np.inf
    return s, k_head.shape[0]


def attention_forward(q, k, v, causal: bool, scale: float, rows=None, window=None):
    """Sparse Query Attention output and log-sum-exp.

    q: [B, N, H_q, d]; k, v: [B, N_kv, H_kv, d] (float64 arrays; N_kv = N
    for self-attention, any length for cross / memory attention, which is
    never causal).
    rows: optional 1-D array of query token indices; all rows when None.
    window: optional (left, right): query t sees only keys
    t - left <= u <= t + right (self-attention only; every row keeps at
    least key t).
    Returns o [B, R, H_q, d] and lse [B, H_q, R] (R = number of rows), with
        o[b,t,h]   = sum_u softmax_u(s_tu) v[b,u,j],  j = h // G
        lse[b,h,t] = log sum_u exp(s_tu)
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, N, H_q, d = q.shape
    H_kv = k.shape[2]
    G = _check_heads(H_q, H_kv)
    _check_lengths(N, k.shape[1], causal)
    window = _check_window(window, N, k.shape[1])
    t_all = np.arange(N) if rows is None else np.asarray(rows, dtype=np.int64)
    R = t_all.shape[0]
    o = np.empty((B, R, H_q, d), dtype=np.float64)
    lse = np.empty((B, H_q, R), dtype=np.float64)
    for b in range(B):
        for h in range(H_q):
            j = h // G
            for c0 in range(0, R, _CHUNK):
                t = t_all[c0:c0 + _CHUNK]
                s, n_keys = _scores(q[b, t, h, :], k[b, :, j, :], t, causal, scale, window)
                m = s.max(axis=1, keepdims=True)
                w = np.exp(s - m)
                l = w.sum(axis=1)
                o[b, c0:c0 + len(t), h, :] = (w @ v[b, :n_keys, j, :]) / l[:, None]
                lse[b, h, c0:c0 + len(t)] = m[:, 0] + np.log(l)
    return o, lse


def attention_backward(q, k, v, do, causal: bool, scale: float, window=None):
    """Gradients of L = sum(o * do) with respect to q, k and v.

    Chain rule through the definition above, per (b, h) with j = h // G:
        P   = softmax rows of s
        dP  = do_h v_j^T
        dS  = P * (dP - rowsum(P * dP))      (softmax Jacobian)
        dq_h  = scale * dS k_j
        dk_j += scale * dS^T q_h             (summed over the G heads of group j)
        dv_j += P^T do_h                     (summed over the G heads of group j)
    with P zero outside the causal mask / window, as in attention_forward.
    Returns dq [B,N,H_q,d], dk and dv [B,N,H_kv,d].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    B, N, H_q, d = q.shape
    H_kv = k.shape[2]
    G = _check_heads(H_q, H_kv)
    _check_lengths(N, k.shape[1], causal)
    window = _check_window(window, N, k.shape[1])
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    t_all = np.arange(N)
    for b in range(B):
        for h in range(H_q):
            j = h // G
            for c0 in range(0, N, _CHUNK):
                t = t_all[c0:c0 + _CHUNK]
                s, n_keys = _scores(q[b, t, h, :], k[b, :, j, :], t, causal, scale, window)
                m = s.max(axis=1, keepdims=True)
                w = np.exp(s - m)
                p = w / w.sum(axis=1, keepdims=True)
                g = do[b, t, h, :]
                dp = g @ v[b, :n_keys, j, :].T
                ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
                dq[b, t, h, :] = scale * (ds @ k[b, :n_keys, j, :])
                dk[b, :n_keys, j, :] += scale * (ds.T @ q[b, t, h, :])
                dv[b, :n_keys, j, :] += p.T @ g
    return dq, dk, dv


def attention_decode(q, k_cache, v_cache, cache_lens, scale: float):
    """Decoding against a key/value cache: autoregressive inference, whose
    latency the abstract of "Sparse Query Attention (SQA): ..." describes as
    bound by memory bandwidth (the regime MQA/GQA address by sharing K/V),
    unlike the compute-bound training and full-sequence work SQA targets.

    q: [B, n_new, H_q, d], the queries of the last n_new tokens of each
    sequence; k_cache, v_cache: [B, L_max, H_kv, d], of which the first
    cache_lens[b] tokens of sequence b are valid (the new tokens' keys and
    values included, so n_new <= cache_lens[b] <= L_max); the rest is never
    read.  Token i of sequence b sits at position p = cache_lens[b] - n_new + i
    and sees keys 0..p (the causal rule).
    Returns o [B, n_new, H_q, d] and lse [B, H_q, n_new].
    """
    q = np.asarray(q, dtype=np.float64)
    B, n_new, H_q, d = q.shape
    H_kv = k_cache.shape[2]
    G = _check_heads(H_q, H_kv)
    L_max = k_cache.shape[1]
    o = np.empty((B, n_new, H_q, d), dtype=np.float64)
    lse = np.empty((B, H_q, n_new), dtype=np.float64)
    for b in range(B):
        L = int(cache_lens[b])
        if not n_new <= L <= L_max:
            raise ValueError(f"cache length {L} outside [{n_new}, {L_max}]")
        k = np.asarray(k_cache[b, :L], dtype=np.float64)
        v = np.asarray(v_cache[b, :L], dtype=np.float64)
        pos = L - n_new + np.arange(n_new)
        for h in range(H_q):
            j = h // G
            s = scale * (q[b, :, h, :] @ k[:, j, :].T)
            s[np.arange(L)[None, :] > pos[:, None]] = -np.inf
            m = s.max(axis=1, keepdims=True)
            w = np.exp(s - m)
            l = w.sum(axis=1)
            o[b, :, h, :] = (w @ v[:, j, :]) / l[:, None]
            lse[b, h, :] = m[:, 0] + np.log(l)
    return o, lse


def projection(x, w, bias=None):
    """y = x w^T (+ bias): x [M, K], w [Nout, K] in nn.Linear layout."""
    y = np.asarray(x, dtype=np.float64) @ np.asarray(w, dtype=np.float64).T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y


def sqa_layer_forward(x, wq, wk, wv, wo, B: int, N: int, H_q: int, H_kv: int,
                      d_head: int, causal: bool = True, scale=None):
    """One SQA attention layer: reduced-width Q/K/V projections, the
    attention core, and the output projection from H_q*d_head back to
    d_model.  All in fp64 with no intermediate rounding.

    x [B*N, d_model]; wq [H_q*d, d_model]; wk, wv [H_kv*d, d_model];
    wo [d_model, H_q*d].  Returns a dict with q, k, v, o (attention output,
    [B*N, H_q*d]) and y [B*N, d_model].
    """
    if scale is None:
        scale = 1.0 / np.sqrt(d_head)
    q = projection(x, wq).reshape(B, N, H_q, d_head)
    k = projection(x, wk).reshape(B, N, H_kv, d_head)
    v = projection(x, wv).reshape(B, N, H_kv, d_head)
    o, lse = attention_forward(q, k, v, causal, scale)
    o2 = o.reshape(B * N, H_q * d_head)
    y = projection(o2, wo)
    return {"q": q, "k": k, "v": v, "o": o2, "lse": lse, "y": y}


def projection_backward(x, w, dy):
    """Gradients of L = sum(y * dy) for y = x w^T: dx = dy w, dw = dy^T x."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    return dy @ w, dy.T @ x


def sqa_layer_backward(x, wq, wk, wv, wo, dy, B: int, N: int, H_q: int, H_kv: int,
                       d_head: int, causal: bool = True, scale=None):
    """Gradient of the SQA layer above for L = sum(y * dy), all in fp64:
    output projection, attention core (attention_backward), then the three
    reduced-width input projections, whose input gradients add up in dx.
    Returns dx [B*N, d_model], dwq, dwk, dwv, dwo (shapes of the weights)."""
    if scale is None:
        scale = 1.0 / np.sqrt(d_head)
    fwd = sqa_layer_forward(x, wq, wk, wv, wo, B, N, H_q, H_kv, d_head, causal, scale)
    do2, dwo = projection_backward(fwd["o"], wo, dy)
    dq, dk, dv = attention_backward(fwd["q"], fwd["k"], fwd["v"], do2.reshape(B, N, H_q, d_head), causal, scale)
    dxq, dwq = projection_backward(x, wq, dq.reshape(B * N, H_q * d_head))
    dxk, dwk = projection_backward(x, wk, dk.reshape(B * N, H_kv * d_head))
    dxv, dwv = projection_backward(x, wv, dv.reshape(B * N, H_kv * d_head))
    return {"dx": dxq + dxk + dxv, "dwq": dwq, "dwk": dwk, "dwv": dwv, "dwo": dwo}
