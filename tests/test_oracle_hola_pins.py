"""Pins of the surprise-cache read oracle (A Hippocampus for Linear Attention, sections 3.3-3.4).

Each compares the token-by-token oracle with another route to the same quantity: full causal softmax
attention in matrix form (the page's Eq. (4) instance), an online cache kept with evictions, the sink's
closed-form damping, the RMSNorm scale, and the near-argmax retrieval the page claims.
"""

import heapq

import numpy as np
import pytest

from oracle import hola_cache_read, rms_norm, top_w_indices


def _inputs(seed, B=1, H=2, L=40, dk=8, dv=5):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, L, dk))
    k = rng.standard_normal((B, H, L, dk))
    v = rng.standard_normal((B, H, L, dv))
    m = rng.random((B, H, L))
    gq = 0.5 + rng.random(dk)
    gk = 0.5 + rng.random(dk)
    sink = rng.standard_normal(H)
    return q, k, v, m, gq, gk, sink


def test_cache_holding_all_history_is_causal_softmax_attention():
    """With w >= L every earlier token stays visible and a sink at -inf adds nothing: the read is
    full causal softmax attention of the normalised q, k (the page's Eq. (4) instance)."""
    q, k, v, m, gq, gk, _ = _inputs(1, L=37)
    dk = q.shape[-1]
    res = hola_cache_read(q, k, v, m, gq, gk, sink=np.full(2, -1e30), w=64, block=8)
    Q, K = rms_norm(q, gq), rms_norm(k, gk)
    logits = np.einsum("bhtd,bhjd->bhtj", Q, K) / np.sqrt(dk)
    L = q.shape[2]
    logits = np.where(np.tril(np.ones((L, L), dtype=bool)), logits, -np.inf)
    p = np.exp(logits - logits.max(-1, keepdims=True))
    p /= p.sum(-1, keepdims=True)
    np.testing.assert_allclose(res["o"], np.einsum("bhtj,bhjd->bhtd", p, v), rtol=1e-12, atol=1e-13)


def test_online_cache_equals_blockwise_top_w():
    """The page: the top-w set can be kept online or selected blockwise without order dependence.
    Keep it online with a min-heap (evict the smallest m, the later token first on ties)."""
    rng = np.random.default_rng(2)
    L, w = 500, 64
    m = rng.random(L)
    m[[50, *range(100, 110), 300, 450]] = np.sort(m)[::-1][58]  # eleven-plus ties that straddle the cut
    heap = []
    for t in range(L):
        heapq.heappush(heap, (m[t], -t))
        if len(heap) > w:
            heapq.heappop(heap)
        if t % 64 == 63 or t == L - 1:
            online = sorted(-j for _, j in heap)
            assert online == top_w_indices(m, t + 1, w)


def test_sink_only_damps_the_read():
    """The null sink carries no value: o(sink) = o(no sink) * Z / (Z + exp(sink))."""
    q, k, v, m, gq, gk, sink = _inputs(3, L=30)
    no = hola_cache_read(q, k, v, m, gq, gk, sink=np.full(2, -1e30), w=8, block=8)
    yes = hola_cache_read(q, k, v, m, gq, gk, sink=sink, w=8, block=8)
    dk = q.shape[-1]
    Q, K = rms_norm(q, gq), rms_norm(k, gk)
    for h in range(2):
        for t in range(30):
            b0 = (t // 8) * 8
            vis = top_w_indices(m[0, h], b0, 8) + list(range(b0, t + 1))
            Z = np.exp(np.array([Q[0, h, t] @ K[0, h, j] for j in vis]) / np.sqrt(dk)).sum()
            np.testing.assert_allclose(yes["o"][0, h, t], no["o"][0, h, t] * Z / (Z + np.exp(sink[h])),
                                       rtol=1e-12, atol=1e-14)


def test_rms_norm_scale():
    """RMSNorm with a constant gamma has root-mean-square |gamma| (up to eps): with gamma = 1 a
    head-dim-d vector has norm sqrt(d), the sharpening the page relies on."""
    rng = np.random.default_rng(4)
    x = rng.standard_normal((5, 128)) * 3.0
    y = rms_norm(x, np.full(128, 2.0), eps=0.0)
    np.testing.assert_allclose(np.sqrt((y * y).mean(-1)), 2.0, rtol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(rms_norm(x, np.ones(128), eps=0.0), axis=-1), np.sqrt(128), rtol=1e-12)


def test_sharpened_read_retrieves_the_matching_cached_value():
    """Near-argmax retrieval (page, section 3.4): with the sqrt(d)-norm logits a query equal to a cached
    key takes almost all the mass among orthogonal keys, so the read returns that key's value."""
    d, L = 128, 128
    rng = np.random.default_rng(5)
    k = np.linalg.qr(rng.standard_normal((d, d)))[0].T[None, None]  # orthonormal keys
    v = rng.standard_normal((1, 1, L, 4))
    m = rng.random((1, 1, L))
    m[0, 0, 10] = 5.0                        # token 10 is the most surprising: cached
    q = np.zeros((1, 1, L, d))
    q[0, 0, 120] = k[0, 0, 10] * 4.0         # token 120 (block 1) queries the cached key of token 10
    res = hola_cache_read(q, k, v, m, np.full(d, 3.0), np.full(d, 3.0), sink=np.array([-1e30]), w=8, block=64)
    np.testing.assert_allclose(res["o"][0, 0, 120], v[0, 0, 10], atol=1e-3)
    assert 10 in res["cache"][0, 0]


def test_reads_are_causal_and_the_cache_comes_from_earlier_blocks():
    q, k, v, m, gq, gk, sink = _inputs(6, L=48)
    base = hola_cache_read(q, k, v, m, gq, gk, sink=sink, w=6, block=16)
    v2, m2 = v.copy(), m.copy()
    v2[:, :, 21] += 10.0   # a later token of block 1
    m2[:, :, 17] += 10.0   # surprise of a token of block 1 (enters the cache only for block 2)
    res = hola_cache_read(q, k, v2, m2, gq, gk, sink=sink, w=6, block=16)
    np.testing.assert_array_equal(res["o"][:, :, :21], base["o"][:, :, :21])
    assert not np.allclose(res["o"][:, :, 32:], base["o"][:, :, 32:])
