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


def _riccati_token_map(a, qn, k, r):
    """The full-covariance step P -> P^- (I + k k^T P^- / r)^-1 with P^- = a^2 P + Qn I, as the 2d x 2d
    transfer matrix of the homogeneous pair P = X Y^-1: [X; Y] -> M [X; Y]."""
    d = k.shape[0]
    eye = np.eye(d)
    kk = np.outer(k, k) / r
    return np.block([[a * a * eye, qn * eye], [a * a * kk, qn * kk + eye]])


@pytest.mark.parametrize("seed", [0, 1])
def test_full_covariance_riccati_composes_as_segment_transfer_matrices(seed):
    """The dense covariance recursion is a matrix Moebius (linear-fractional) map of P (Kalman Delta
    Networks, Abstract): each token multiplies the homogeneous pair [X; Y] (P = X Y^-1) by a 2d x 2d matrix,
    so a segment's map is the product of its tokens' matrices, renormalised by any scalar.  Chaining the
    segment maps from P0 gives the oracle's P at every segment boundary; a wrong block (a instead of a^2,
    the update's k k^T / r in the upper right, Qn missing from the lower right) fails it."""
    d, L, seg = 6, 96, 16
    x = _inputs(seed, L, d)
    P0 = np.eye(d) * 0.7 + 0.05
    ref = scan_kalman_full(x["q"], x["k"], x["v"], x["r"], a=x["a"], qn=x["qn"], P0=P0, return_states=True)
    X, Y = P0.copy(), np.eye(d)
    for lo in range(0, L, seg):
        M = np.eye(2 * d)
        for t in range(lo, lo + seg):
            M = _riccati_token_map(x["a"][t], x["qn"][t], x["k"][t], x["r"][t]) @ M
            M = M / np.abs(M).max()
        XY = M @ np.vstack([X, Y])
        X, Y = XY[:d], XY[d:]
        P = X @ np.linalg.inv(Y)
        np.testing.assert_allclose(P, ref["P_hist"][lo + seg - 1], rtol=0, atol=1e-10)
        np.testing.assert_allclose(P, P.T, atol=1e-10)


def _riccati_chunk_map(a, qn, k, r):
    """Closed form of the product M_C ... M_1 of a chunk's token transfer matrices.

    M_t = D_t + u_t v_t^T with D_t = [[a_t^2 I, Qn_t I], [0, I]], u_t = [0; k_t], v_t = [a_t^2 k_t; Qn_t k_t] / r_t,
    so the product is [[alpha I, beta I], [0, I]] + U W^T with alpha = prod a^2, beta = the accumulated
    process noise, column j of U = [beta_{C,j} k_j; k_j] (beta_{t,j}: the noise accumulated over tokens
    j+1..t) and W = B (diag(r) - Cs^T)^-1, where column t of B is [alpha_t k_t; beta_t k_t] and
    Cs_tj = (k_j . k_t) beta_{t,j} for j < t: one triangular solve of the chunk's size."""
    C, d = k.shape
    alpha = np.cumprod(a * a)                     # alpha_t
    beta = np.zeros(C)                            # beta_t = a_t^2 beta_{t-1} + Qn_t
    for t in range(C):
        beta[t] = a[t] ** 2 * (beta[t - 1] if t else 0.0) + qn[t]
    bt = np.zeros((C, C))                         # beta_{t,j}, j <= t (beta_{j,j} = 0)
    for j in range(C):
        acc = 0.0
        for t in range(j + 1, C):
            acc = a[t] ** 2 * acc + qn[t]
            bt[t, j] = acc
    Cs = np.tril((k @ k.T) * bt, -1)
    Bm = np.vstack([alpha[None, :] * k.T, beta[None, :] * k.T])       # 2d x C
    W = np.linalg.solve((np.diag(r) - Cs.T).T, Bm.T).T                # B (diag(r) - Cs^T)^-1
    U = np.vstack([bt[C - 1][None, :] * k.T, k.T])
    eye = np.eye(d)
    return np.block([[alpha[-1] * eye, beta[-1] * eye], [0 * eye, eye]]) + U @ W.T


@pytest.mark.parametrize("seed", [0, 3])
def test_riccati_chunk_transfer_matrix_in_closed_form(seed):
    """The closed form above equals the product of the chunk's token matrices (a chunk-parallel covariance
    side can build every chunk's map at once and only chain the maps)."""
    d, C = 5, 12
    x = _inputs(seed, C, d)
    M = np.eye(2 * d)
    for t in range(C):
        M = _riccati_token_map(x["a"][t], x["qn"][t], x["k"][t], x["r"][t]) @ M
    np.testing.assert_allclose(_riccati_chunk_map(x["a"], x["qn"], x["k"], x["r"]), M, rtol=1e-11, atol=1e-12)


def _riccati_chunk_apply_gform(a, qn, k, r, X, Y):
    """The chunk map applied to [X; Y] without forming W: with G = (diag(r) - Cs^T)^-1, whose row j follows
    g_jt = (delta_jt + sum_{m<t} g_jm Cs_tm) / r_t, the rank-C term is U Z with
    Z = G^T (diag(alpha_t) K X + diag(beta_t) K Y), so that X' = alpha X + beta Y + K^T diag(beta_{C,j}) Z and
    Y' = Y + K^T Z.  This is the order in which the chain kernel applies a chunk."""
    C, d = k.shape
    alpha = np.cumprod(a * a)
    beta = np.zeros(C)
    for t in range(C):
        beta[t] = a[t] ** 2 * (beta[t - 1] if t else 0.0) + qn[t]
    bt = np.zeros((C, C))
    for j in range(C):
        acc = 0.0
        for t in range(j + 1, C):
            acc = a[t] ** 2 * acc + qn[t]
            bt[t, j] = acc
    Cs = np.tril((k @ k.T) * bt, -1)
    G = np.zeros((C, C))
    for j in range(C):          # row j of G by the forward recurrence
        for t in range(C):
            G[j, t] = ((1.0 if t == j else 0.0) + G[j, :t] @ Cs[t, :t]) / r[t]
    R = alpha[:, None] * (k @ X) + beta[:, None] * (k @ Y)
    Z = G.T @ R
    u = bt[C - 1]
    return alpha[-1] * X + beta[-1] * Y + k.T @ (u[:, None] * Z), Y + k.T @ Z


@pytest.mark.parametrize("seed", [0, 5])
def test_riccati_chunk_map_applied_in_g_form(seed):
    """The G form of a chunk's map (the chain kernel's arithmetic), with G from its row recurrence rather than
    an inverse, equals the product of the chunk's token transfer matrices applied to [X; Y]."""
    d, C, n = 5, 12, 4
    x = _inputs(seed, C, d)
    rng = np.random.default_rng(seed + 100)
    X, Y = rng.standard_normal((d, n)), np.eye(d)[:, :n] + 0.1 * rng.standard_normal((d, n))
    M = np.eye(2 * d)
    for t in range(C):
        M = _riccati_token_map(x["a"][t], x["qn"][t], x["k"][t], x["r"][t]) @ M
    ref = M @ np.vstack([X, Y])
    Xn, Yn = _riccati_chunk_apply_gform(x["a"], x["qn"], x["k"], x["r"], X, Y)
    np.testing.assert_allclose(np.vstack([Xn, Yn]), ref, rtol=1e-11, atol=1e-12)
