"""Pins of the float64 backwards of the four scans (oracle/backward.py), CPU only.

The backward is checked against routes that do not use its reverse recurrence: central finite differences
of the forward oracle for every input, the closed form of the delta scan when nothing is written (beta = 0,
so S_t = A_t S_0 and every output is linear in S_0 and q), a one-token derivation, and the closed form of
the diagonal variances at a = 1, Q = 0.  Shapes use d_k != d_v, q != k, gates below one
and a non-zero start state, so that a transposed product, a missing decay or a dropped path through the
residual fails.
"""

import numpy as np
import pytest

from oracle import scan_delta, scan_kalman_diag, scan_kalman_full, scan_kalman_iso
from oracle.backward import (scan_delta_backward, scan_kalman_diag_backward, scan_kalman_full_backward,
                             scan_kalman_iso_backward)


def _inputs(seed, heads, L, dk, dv):
    rng = np.random.default_rng(seed)
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    x = {
        "q": unit(rng.standard_normal((heads, L, dk))),
        "k": unit(rng.standard_normal((heads, L, dk))) * (1.0 + 0.3 * rng.random((heads, L, 1))),
        "v": rng.standard_normal((heads, L, dv)),
        "beta": 0.2 + 0.7 * rng.random((heads, L)),
        "a": 0.6 + 0.39 * rng.random((heads, L)),
        "S0": 0.5 * rng.standard_normal((heads, dk, dv)),
    }
    up = {"dO": rng.standard_normal((heads, L, dv)), "dm": rng.standard_normal((heads, L)),
          "dS_L": rng.standard_normal((heads, dk, dv))}
    return x, up


def _loss(x, up):
    out = scan_delta(x["q"], x["k"], x["v"], x["beta"], a=x["a"], S0=x["S0"])
    return float(np.sum(up["dO"] * out["o"]) + np.sum(up["dm"] * out["m"]) + np.sum(up["dS_L"] * out["S"]))


@pytest.mark.parametrize("use_dm", [False, True])
def test_backward_matches_central_differences_for_every_input(use_dm):
    x, up = _inputs(3, heads=2, L=9, dk=3, dv=4)
    if not use_dm:
        up["dm"] = np.zeros_like(up["dm"])
    g = scan_delta_backward(x["q"], x["k"], x["v"], x["beta"], up["dO"], a=x["a"], S0=x["S0"], dm=up["dm"],
                            dS_L=up["dS_L"])
    names = {"q": "dq", "k": "dk", "v": "dv", "beta": "dbeta", "a": "da", "S0": "dS0"}
    h = 1e-6
    for name, gname in names.items():
        num = np.zeros_like(x[name])
        it = np.nditer(x[name], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = {kk: vv.copy() for kk, vv in x.items()}
            xm = {kk: vv.copy() for kk, vv in x.items()}
            xp[name][idx] += h
            xm[name][idx] -= h
            num[idx] = (_loss(xp, up) - _loss(xm, up)) / (2 * h)
        scale = np.abs(num).max()
        assert np.abs(g[gname] - num).max() <= 1e-6 * max(scale, 1.0), (name, np.abs(g[gname] - num).max(), scale)


def test_backward_without_writes_is_the_closed_form():
    """beta = 0: S_t = A_t S_0 with A_t = a_1 ... a_t, so o_t = A_t S_0^T q_t, and
    dq_t = A_t S_0 dO_t,  dS_0 = sum_t A_t q_t dO_t^T + A_L dS_L,  dv_t = 0,
    da_t = (1 / a_t) sum_{s >= t} A_s <q_s dO_s^T, S_0> + (A_L / a_t) <dS_L, S_0>."""
    x, up = _inputs(5, heads=1, L=7, dk=3, dv=2)
    x["beta"] = np.zeros_like(x["beta"])
    g = scan_delta_backward(x["q"], x["k"], x["v"], x["beta"], up["dO"], a=x["a"], S0=x["S0"], dS_L=up["dS_L"])
    a, q, dO, S0, dSL = x["a"][0], x["q"][0], up["dO"][0], x["S0"][0], up["dS_L"][0]
    A = np.cumprod(a)
    np.testing.assert_allclose(g["dq"][0], A[:, None] * (dO @ S0.T), rtol=1e-12, atol=1e-14)
    dS0 = sum(A[t] * np.outer(q[t], dO[t]) for t in range(7)) + A[-1] * dSL
    np.testing.assert_allclose(g["dS0"][0], dS0, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(g["dv"][0], 0.0, atol=1e-15)
    read = np.array([A[s] * np.sum(np.outer(q[s], dO[s]) * S0) for s in range(7)])
    da = np.array([(read[t:].sum() + A[-1] * np.sum(dSL * S0)) / a[t] for t in range(7)])
    np.testing.assert_allclose(g["da"][0], da, rtol=1e-12, atol=1e-14)


def test_backward_of_a_single_token_by_hand():
    """One token from S_0 = 0 with a = 1: S_1 = beta k v^T, o = beta (q.k) v, so
    dq = beta (v.dO) k, dv = beta (q.k) dO, dbeta = (q.k)(v.dO), dk = beta (v.dO) q."""
    rng = np.random.default_rng(7)
    q, k, v, dO = rng.standard_normal(3), rng.standard_normal(3), rng.standard_normal(2), rng.standard_normal(2)
    b = 0.7
    g = scan_delta_backward(q[None], k[None], v[None], np.array([b]), dO[None])
    np.testing.assert_allclose(g["dq"][0], b * (v @ dO) * k, rtol=1e-13)
    np.testing.assert_allclose(g["dv"][0], b * (q @ k) * dO, rtol=1e-13)
    np.testing.assert_allclose(g["dbeta"][0], (q @ k) * (v @ dO), rtol=1e-13)
    np.testing.assert_allclose(g["dk"][0], b * (v @ dO) * q, rtol=1e-13)


# ----------------------------------------------------------------------------- diagonal Kalman


def _diag_inputs(seed, heads, L, dk, dv):
    rng = np.random.default_rng(seed)
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    x = {
        "q": unit(rng.standard_normal((heads, L, dk))),
        "k": unit(rng.standard_normal((heads, L, dk))) * (1.0 + 0.3 * rng.random((heads, L, 1))),
        "v": rng.standard_normal((heads, L, dv)),
        "r": 0.3 + rng.random((heads, L)),
        "a": 0.6 + 0.39 * rng.random((heads, L)),
        "qn": 0.05 * rng.random((heads, L)),
        "S0": 0.5 * rng.standard_normal((heads, dk, dv)),
        "p0": 0.5 + rng.random((heads, dk)),
    }
    up = {"dO": rng.standard_normal((heads, L, dv)), "dm": rng.standard_normal((heads, L)),
          "dS_L": rng.standard_normal((heads, dk, dv)), "dp_L": rng.standard_normal((heads, dk))}
    return x, up


def _diag_loss(x, up):
    out = scan_kalman_diag(x["q"], x["k"], x["v"], x["r"], a=x["a"], qn=x["qn"], S0=x["S0"], p0=x["p0"])
    return float(np.sum(up["dO"] * out["o"]) + np.sum(up["dm"] * out["m"]) + np.sum(up["dS_L"] * out["S"])
                 + np.sum(up["dp_L"] * out["p"]))


def test_diagonal_kalman_backward_matches_central_differences_for_every_input():
    x, up = _diag_inputs(11, heads=2, L=8, dk=3, dv=4)
    g = scan_kalman_diag_backward(x["q"], x["k"], x["v"], x["r"], up["dO"], a=x["a"], qn=x["qn"], S0=x["S0"],
                                  p0=x["p0"], dm=up["dm"], dS_L=up["dS_L"], dp_L=up["dp_L"])
    names = {"q": "dq", "k": "dk", "v": "dv", "r": "dr", "a": "da", "qn": "dqn", "S0": "dS0", "p0": "dp0"}
    h = 1e-6
    for name, gname in names.items():
        num = np.zeros_like(x[name])
        it = np.nditer(x[name], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = {kk: vv.copy() for kk, vv in x.items()}
            xm = {kk: vv.copy() for kk, vv in x.items()}
            xp[name][idx] += h
            xm[name][idx] -= h
            num[idx] = (_diag_loss(xp, up) - _diag_loss(xm, up)) / (2 * h)
        scale = np.abs(num).max()
        assert np.abs(g[gname] - num).max() <= 1e-6 * max(scale, 1.0), (name, np.abs(g[gname] - num).max(), scale)


def test_diagonal_kalman_backward_of_the_variances_alone():
    """With only dp_L upstream and a = 1, Q = 0 the variances have the closed form
    1 / p_L,i = 1 / p_0,i + sum_t k_ti^2 / r_t, so dp0_i = dp_L,i p_L,i^2 / p_0,i^2 and
    dr_t = sum_i dp_L,i p_L,i^2 k_ti^2 / r_t^2 (S, o and m do not reach the loss)."""
    x, up = _diag_inputs(13, heads=1, L=6, dk=3, dv=2)
    zero = np.zeros_like
    g = scan_kalman_diag_backward(x["q"], x["k"], x["v"], x["r"], zero(up["dO"]), p0=x["p0"], dp_L=up["dp_L"])
    pL = scan_kalman_diag(x["q"], x["k"], x["v"], x["r"], p0=x["p0"])["p"][0]
    p0, k, r, dpL = x["p0"][0], x["k"][0], x["r"][0], up["dp_L"][0]
    np.testing.assert_allclose(g["dp0"][0], dpL * pL ** 2 / p0 ** 2, rtol=1e-12)
    np.testing.assert_allclose(g["dr"][0], ((dpL * pL ** 2)[None, :] * k ** 2).sum(-1) / r ** 2, rtol=1e-12)


# ----------------------------------------------------------------------------- isotropic and full Kalman


def _central_differences(loss, x, names):
    h = 1e-6
    out = {}
    for name in names:
        num = np.zeros_like(x[name])
        it = np.nditer(x[name], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = {kk: vv.copy() for kk, vv in x.items()}
            xm = {kk: vv.copy() for kk, vv in x.items()}
            xp[name][idx] += h
            xm[name][idx] -= h
            num[idx] = (loss(xp) - loss(xm)) / (2 * h)
        out[name] = num
    return out


def _assert_close(g, num, names):
    for name, gname in names.items():
        scale = np.abs(num[name]).max()
        err = np.abs(g[gname] - num[name]).max()
        assert err <= 1e-6 * max(scale, 1.0), (name, err, scale)


def test_isotropic_kalman_backward_matches_central_differences_for_every_input():
    x, up = _diag_inputs(17, heads=2, L=8, dk=3, dv=4)
    x["c0"] = 0.5 + np.random.default_rng(18).random(2)
    del x["p0"]
    dcL = np.random.default_rng(19).standard_normal(2)

    def loss(xx):
        out = scan_kalman_iso(xx["q"], xx["k"], xx["v"], xx["r"], a=xx["a"], qn=xx["qn"], S0=xx["S0"], c0=xx["c0"])
        return float(np.sum(up["dO"] * out["o"]) + np.sum(up["dm"] * out["m"]) + np.sum(up["dS_L"] * out["S"])
                     + np.sum(dcL * out["c"]))

    g = scan_kalman_iso_backward(x["q"], x["k"], x["v"], x["r"], up["dO"], a=x["a"], qn=x["qn"], S0=x["S0"],
                                 c0=x["c0"], dm=up["dm"], dS_L=up["dS_L"], dc_L=dcL)
    names = {"q": "dq", "k": "dk", "v": "dv", "r": "dr", "a": "da", "qn": "dqn", "S0": "dS0", "c0": "dc0"}
    _assert_close(g, _central_differences(loss, x, names), names)


def test_full_kalman_backward_matches_central_differences_for_every_input():
    x, up = _diag_inputs(21, heads=2, L=7, dk=3, dv=4)
    rng = np.random.default_rng(22)
    B = rng.standard_normal((2, 3, 3)) / 3
    x["P0"] = 0.5 * np.eye(3) + B @ np.swapaxes(B, 1, 2)
    del x["p0"]
    dPL = rng.standard_normal((2, 3, 3))

    def loss(xx):
        out = scan_kalman_full(xx["q"], xx["k"], xx["v"], xx["r"], a=xx["a"], qn=xx["qn"], S0=xx["S0"], P0=xx["P0"])
        return float(np.sum(up["dO"] * out["o"]) + np.sum(up["dm"] * out["m"]) + np.sum(up["dS_L"] * out["S"])
                     + np.sum(dPL * out["P"]))

    g = scan_kalman_full_backward(x["q"], x["k"], x["v"], x["r"], up["dO"], a=x["a"], qn=x["qn"], S0=x["S0"],
                                  P0=x["P0"], dm=up["dm"], dS_L=up["dS_L"], dP_L=dPL)
    names = {"q": "dq", "k": "dk", "v": "dv", "r": "dr", "a": "da", "qn": "dqn", "S0": "dS0", "P0": "dP0"}
    _assert_close(g, _central_differences(loss, x, names), names)


def test_full_kalman_backward_equals_diagonal_backward_on_one_hot_keys():
    """One-hot keys and a diagonal P0 keep the full covariance diagonal, and the two filters coincide
    (a pin of the forwards); their gradients with respect to q, v, r, a, Qn, S0 and the start variances
    must then coincide as well."""
    rng = np.random.default_rng(23)
    L, dk, dv = 9, 4, 3
    idx = rng.integers(0, dk, L)
    k = np.eye(dk)[idx][None]
    q = rng.standard_normal((1, L, dk))
    v = rng.standard_normal((1, L, dv))
    r, a, qn = 0.3 + rng.random((1, L)), 0.6 + 0.39 * rng.random((1, L)), 0.05 * rng.random((1, L))
    S0, p0 = rng.standard_normal((1, dk, dv)), 0.5 + rng.random((1, dk))
    dO, dm, dSL = rng.standard_normal((1, L, dv)), rng.standard_normal((1, L)), rng.standard_normal((1, dk, dv))
    gf = scan_kalman_full_backward(q, k, v, r, dO, a=a, qn=qn, S0=S0, P0=p0[:, :, None] * np.eye(dk), dm=dm,
                                   dS_L=dSL)
    gd = scan_kalman_diag_backward(q, k, v, r, dO, a=a, qn=qn, S0=S0, p0=p0, dm=dm, dS_L=dSL)
    for key in ("dq", "dv", "dr", "da", "dqn", "dS0"):
        np.testing.assert_allclose(gf[key], gd[key], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(np.diagonal(gf["dP0"], axis1=1, axis2=2), gd["dp0"], rtol=1e-10, atol=1e-12)
