"""The two facts the segment-parallel scans stand on, checked on the float64 oracle (CPU).

Kalman Delta Networks, Abstract: the uncertainty recurrences of the diagonal and isotropic variants are
Moebius maps, which is what lets a sequence be cut into pieces whose maps compose.  And once the gains
are fixed, the memory scan over a piece sends its start state S0 to M S0 + B.  These tests cut the
oracle's sequence into segments, compose per-coordinate 2x2 maps to get the uncertainty at every segment
start, take each segment's affine map from two oracle runs (S0 = 0 and S0 = I), chain the maps, rerun
the segments from the chained states, and compare everything with one uninterrupted oracle run.  A
wrong map entry, a transposed M (d_k = d_v here, and q != k, so M is not symmetric) or an off-by-one
segment boundary fails them.
"""

import numpy as np
import pytest

from oracle import scan_delta, scan_kalman_diag, scan_kalman_full, scan_kalman_iso


def _unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _inputs(seed, L, d):
    rng = np.random.default_rng(seed)
    return {
        "q": _unit_rows(rng.standard_normal((L, d))),
        "k": _unit_rows(rng.standard_normal((L, d))),
        "v": rng.standard_normal((L, d)),
        "beta": 1.0 / (1.0 + np.exp(-rng.standard_normal(L))),
        "a": np.exp(-np.log1p(np.exp(rng.standard_normal(L) - 2.0))),
        "r": np.log1p(np.exp(rng.standard_normal(L))) + 0.1,
        "qn": 1e-3 * (1.0 + rng.random(L)),
    }


def _token_map(a, qn, w):
    """c -> c^- / (1 + w c^-) with c^- = a^2 c + Qn, as a 2x2 matrix."""
    return np.array([[a * a, qn], [w * a * a, w * qn + 1.0]])


def _apply(M, c):
    return (M[0, 0] * c + M[0, 1]) / (M[1, 0] * c + M[1, 1])


def _segment_map(x, lo, hi, w_of_t):
    M = np.eye(2)
    for t in range(lo, hi):
        M = _token_map(x["a"][t], x["qn"][t], w_of_t(t)) @ M
        M = M / M[1, 1]
    return M


def _run(variant, x, lo, hi, S0, U0):
    sl = slice(lo, hi)
    q, k, v = x["q"][sl], x["k"][sl], x["v"][sl]
    if variant == "delta":
        return scan_delta(q, k, v, x["beta"][sl], a=x["a"][sl], S0=S0)
    if variant == "kalman_diag":
        return scan_kalman_diag(q, k, v, x["r"][sl], a=x["a"][sl], qn=x["qn"][sl], S0=S0, p0=U0)
    if variant == "kalman_iso":
        return scan_kalman_iso(q, k, v, x["r"][sl], a=x["a"][sl], qn=x["qn"][sl], S0=S0, c0=U0)
    return scan_kalman_full(q, k, v, x["r"][sl], a=x["a"][sl], qn=x["qn"][sl], S0=S0, P0=U0)


@pytest.mark.parametrize("L,P", [(48, 4), (50, 5), (45, 3)])
def test_diagonal_uncertainty_at_segment_starts_by_composed_moebius_maps(L, P):
    d = 6
    x = _inputs(1, L, d)
    p0 = 0.5 + np.random.default_rng(2).random(d)
    ref = scan_kalman_diag(x["q"], x["k"], x["v"], x["r"], a=x["a"], qn=x["qn"], p0=p0, return_states=True)
    Ls = L // P
    for i in range(d):
        c = p0[i]
        for s in range(P):
            if s > 0:
                np.testing.assert_allclose(c, ref["p_hist"][s * Ls - 1, i], rtol=1e-12)
            M = _segment_map(x, s * Ls, (s + 1) * Ls, lambda t: x["k"][t, i] ** 2 / x["r"][t])
            c = _apply(M, c)
        np.testing.assert_allclose(c, ref["p"][i], rtol=1e-12)


def test_isotropic_uncertainty_at_segment_starts_by_composed_moebius_maps():
    L, P, d = 60, 4, 5
    x = _inputs(3, L, d)
    ref = scan_kalman_iso(x["q"], x["k"], x["v"], x["r"], a=x["a"], qn=x["qn"], c0=0.7, return_states=True)
    Ls = L // P
    c = 0.7
    for s in range(P):
        if s > 0:
            np.testing.assert_allclose(c, ref["c_hist"][s * Ls - 1], rtol=1e-12)
        c = _apply(_segment_map(x, s * Ls, (s + 1) * Ls,
                                lambda t: np.dot(x["k"][t], x["k"][t]) / (d * x["r"][t])), c)
    np.testing.assert_allclose(c, ref["c"], rtol=1e-12)


@pytest.mark.parametrize("variant", ["delta", "kalman_diag", "kalman_iso", "kalman_full"])
@pytest.mark.parametrize("L,P", [(40, 4), (42, 3)])
def test_segmented_scan_equals_the_serial_scan(variant, L, P):
    d = 5
    x = _inputs(4, L, d)
    rng = np.random.default_rng(5)
    S0 = rng.standard_normal((d, d))
    U0 = {"delta": None, "kalman_diag": 0.5 + rng.random(d), "kalman_iso": 0.8,
          "kalman_full": np.eye(d) * 0.9 + 0.05 * np.ones((d, d))}[variant]
    ref = _run(variant, x, 0, L, S0, U0)
    Ls = L // P
    ukey = {"delta": None, "kalman_diag": "p", "kalman_iso": "c", "kalman_full": "P"}[variant]
    # uncertainty at each segment start (the covariance side does not depend on S)
    starts = [U0]
    for s in range(P - 1):
        starts.append(_run(variant, x, s * Ls, (s + 1) * Ls, np.zeros((d, d)), starts[-1])[ukey] if ukey else None)
    # each segment's affine map S0 -> M S0 + B from two runs
    S = S0
    o, m = [], []
    for s in range(P):
        lo, hi = s * Ls, (s + 1) * Ls
        B = _run(variant, x, lo, hi, np.zeros((d, d)), starts[s])["S"]
        M = _run(variant, x, lo, hi, np.eye(d), starts[s])["S"] - B
        out = _run(variant, x, lo, hi, S, starts[s])
        np.testing.assert_allclose(out["S"], M @ S + B, rtol=1e-10, atol=1e-12)
        o.append(out["o"]), m.append(out["m"])
        S = M @ S + B
    np.testing.assert_allclose(np.concatenate(o), ref["o"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(np.concatenate(m), ref["m"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(S, ref["S"], rtol=1e-10, atol=1e-12)
