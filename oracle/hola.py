"""Float64 CPU oracle for the surprise-cache read of HOLA (test infrastructure only).

TEST INFRASTRUCTURE ONLY, like ``oracle.scan``: the product never imports it.

A Hippocampus for Linear Attention, section 3.3 (what to store) and section 3.4
(how to read), Eq. (6)-(7):

* each head keeps an exact cache of the (k, v) pairs of the w tokens with the
  largest surprise m_t = ||Delta_t||_F seen so far (default w = 64); the set can
  be kept online or selected blockwise with the same result;
* the read of token t is a softmax over the visible set V_t = cache of the
  earlier blocks, the causal tokens of t's own block, and one null sink:
      o_t = sum_{j in V_t} softmax_j(q~_t^T k~_j / sqrt(d)) v_j,
      q~ = RMSNorm_gamma_q(q),  k~ = RMSNorm_gamma_k(k),
  with the temperature fixed to 1.

Readings where the page leaves a step open (kept with the design notes too):

H1  Blocks of ``block`` tokens (default 64, the scan's chunk; the page's runs use
    256).  The cache read by block b holds the top-w tokens of blocks 0..b-1;
    tokens of block b see each other causally (j <= t).
H2  Ties in m are broken towards the earlier token.
H3  RMSNorm(x) = x / sqrt(mean(x^2) + eps) * gamma with eps = 1e-6 (the
    Qwen3-style norm the page names), one gamma per query / key path shared by
    the heads (the page counts 2 d scales per layer).
H4  The null sink is one extra softmax entry per head with logit ``sink[h]``
    and a zero value: it only adds exp(sink) to the denominator.
H5  The read returns o^cache alone; the per-head gate that mixes it with the
    state read (o_t = S_t^T q_t + sigma(g_h) o^cache_t on the page's
    description of a "per-head sink and cache gate") is left to the caller.
"""

from __future__ import annotations

import numpy as np

__all__ = ["rms_norm", "top_w_indices", "hola_cache_read"]


def rms_norm(x, gamma, eps=1e-6):
    """RMSNorm over the last axis (reading H3)."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps) * np.asarray(gamma, dtype=np.float64)


def top_w_indices(m, upto, w):
    """Indices of the (at most) w largest m[0:upto], ties towards the earlier token (reading H2),
    returned in increasing token order."""
    m = np.asarray(m, dtype=np.float64)[:upto]
    order = sorted(range(upto), key=lambda j: (-m[j], j))
    return sorted(order[:w])


def hola_cache_read(q, k, v, m, gamma_q, gamma_k, sink, w=64, block=64, eps=1e-6, tokens=None):
    """Surprise-cache read for q, k [B, H, L, d_k], v [B, H, L, d_v], m [B, H, L], sink [H].

    Token by token: the visible set, the sharpened logits, the softmax with the sink.  ``tokens``
    restricts the read to those token positions (the other rows of o stay 0).
    Returns {"o": [B, H, L, d_v], "cache": [B, H, w] token indices of the final cache (-1 = empty)}.
    """
    q, k, v, m = (np.asarray(x, dtype=np.float64) for x in (q, k, v, m))
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    sink = np.asarray(sink, dtype=np.float64).reshape(H)
    qt = rms_norm(q, gamma_q, eps)
    kt = rms_norm(k, gamma_k, eps)
    o = np.zeros((B, H, L, dv))
    cache_out = -np.ones((B, H, w), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            for t in (range(L) if tokens is None else tokens):
                b0 = (t // block) * block
                vis = top_w_indices(m[b, h], b0, w) + list(range(b0, t + 1))
                logits = np.array([qt[b, h, t] @ kt[b, h, j] for j in vis]) / np.sqrt(dk)
                top = max(logits.max(), sink[h])
                ex = np.exp(logits - top)
                den = ex.sum() + np.exp(sink[h] - top)
                o[b, h, t] = (ex[:, None] * v[b, h, vis]).sum(axis=0) / den
            final = top_w_indices(m[b, h], L, w)
            cache_out[b, h, : len(final)] = final
    return {"o": o, "cache": cache_out}
