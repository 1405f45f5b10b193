"""Pins of the float64 oracle against what the pages and the mathematics fix.

None of these re-types the oracle's own recurrence: each compares it with a
different route to the same quantity (a closed form, explicit Gaussian
conditioning with matrix inverses, autograd, a numerical KL minimisation, a
special case of another variant, or values derived by hand).  Shapes use
d_k != d_v and q != k so that a transposed operand or a swapped read fails.
"""

import json
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import decode_step, kalman_update, scan_delta, scan_kalman_diag, scan_kalman_full, scan_kalman_iso

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _case(seed, L, dk, dv, heads=(1,)):
    rng = np.random.default_rng(seed)
    q = _unit_rows(rng.standard_normal((*heads, L, dk)))
    k = _unit_rows(rng.standard_normal((*heads, L, dk)))
    v = rng.standard_normal((*heads, L, dv))
    return rng, q, k, v


# ----------------------------------------------------------------------------- ridge closed form
# DeltaNet-PC, "How it works": the memory energy is ridge regression on all
# observed pairs, eps/2 ||S||_F^2 + sum_t 1/2 ||v_t - S k_t||^2 (Eq. 5), and the
# RLS update (Eq. 7) is its recursive minimiser.  With a = 1, Q = 0 the Kalman
# filter started from P0 = I/eps with noise r_t is that recursion, so for
# every prefix t: S_t = (eps I + K^T R^-1 K)^-1 K^T R^-1 V and
# P_t = (eps I + K^T R^-1 K)^-1.


@pytest.mark.parametrize("eps,r_kind", [(1.0, "one"), (0.3, "one"), (2.0, "varying")])
def test_kalman_equals_ridge_closed_form_every_prefix(eps, r_kind):
    rng, q, k, v = _case(1, 40, 6, 3)
    L, dk = 40, 6
    r = np.ones(L) if r_kind == "one" else 0.2 + rng.random(L)
    res = scan_kalman_full(q, k, v, r=r[None], P0=(np.eye(dk) / eps)[None], return_states=True)
    for t in range(L):
        K, V, Rinv = k[0, : t + 1], v[0, : t + 1], np.diag(1.0 / r[: t + 1])
        A = eps * np.eye(dk) + K.T @ Rinv @ K
        S_t = np.linalg.solve(A, K.T @ Rinv @ V)
        P_t = np.linalg.inv(A)
        np.testing.assert_allclose(res["S_hist"][0, t], S_t, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(res["P_hist"][0, t], P_t, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(res["o"][0, t], S_t.T @ q[0, t], rtol=1e-10, atol=1e-12)


def test_tiny_workload_kalman_final_state_is_ridge():
    """The tiny fp32 workload (B=1, H=1, L=256, d=16, a=1, Q=0, r=1, P0=I)."""
    torch = pytest.importorskip("torch")
    from delta_rule_recurrent_scan_b200.workloads import WORKLOADS, make_scan_inputs

    w = WORKLOADS["tiny_kalman"]
    x = make_scan_inputs(w, seed=0)
    q, k, v = (x[n].double().numpy() for n in ("q", "k", "v"))
    res = scan_kalman_full(q, k, v, r=x["r"].double().numpy())
    K, V = k[0, 0], v[0, 0]
    S = np.linalg.solve(np.eye(16) + K.T @ K, K.T @ V)
    err = np.abs(res["S"][0, 0] - S).max() / np.abs(S).max()
    assert err < 1e-12
    assert torch.all(x["r"] == 1.0)


# ----------------------------------------------------------------------------- brute-force conditioning
# Kalman Delta Networks, Abstract: the memory is a linear-Gaussian state-space
# model and the Kalman filter its optimal recursive estimator; Memory by
# Design, Abstract: writes are exact Bayesian filtering of mean and covariance.
# Brute force: build the joint Gaussian of (x_0, w_1..w_L, n_1..n_L), map it
# linearly to every x_t and y_t, and condition x_t on y_1..t by explicit
# inverses.  Each column of S is one such state with its own observations.


def _brute_force_posteriors(k, v, a, qn, r, S0, P0):
    L, dk = k.shape
    dv = v.shape[1]
    nz = dk + L * dk + L
    cov_z = np.zeros((nz, nz))
    cov_z[:dk, :dk] = P0
    for t in range(L):
        o = dk + t * dk
        cov_z[o:o + dk, o:o + dk] = qn[t] * np.eye(dk)
        cov_z[dk + L * dk + t, dk + L * dk + t] = r[t]
    Mx = np.zeros((L + 1, dk, nz))
    Mx[0, :, :dk] = np.eye(dk)
    My = np.zeros((L, nz))
    for t in range(L):
        Mx[t + 1] = a[t] * Mx[t]
        Mx[t + 1, :, dk + t * dk: dk + (t + 1) * dk] += np.eye(dk)
        My[t] = k[t] @ Mx[t + 1]
        My[t, dk + L * dk + t] += 1.0
    means, covs = [], []
    for t in range(L):
        Y = My[: t + 1]
        Cyy = Y @ cov_z @ Y.T
        Cxy = Mx[t + 1] @ cov_z @ Y.T
        Cxx = Mx[t + 1] @ cov_z @ Mx[t + 1].T
        G = Cxy @ np.linalg.inv(Cyy)
        Sm = np.zeros((dk, dv))
        for c in range(dv):
            mu_z = np.zeros(nz)
            mu_z[:dk] = S0[:, c]
            y = v[: t + 1, c]
            Sm[:, c] = Mx[t + 1] @ mu_z + G @ (y - Y @ mu_z)
        means.append(Sm)
        covs.append(Cxx - G @ Cxy.T)
    return np.array(means), np.array(covs)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_kalman_full_equals_brute_force_conditioning(seed):
    rng, q, k, v = _case(10 + seed, 9, 4, 3)
    L, dk = 9, 4
    a = 0.3 + 0.7 * rng.random(L)
    qn = 0.05 * rng.random(L)
    r = 0.1 + rng.random(L)
    S0 = rng.standard_normal((dk, 3))
    M = rng.standard_normal((dk, dk))
    P0 = M @ M.T + 0.5 * np.eye(dk)
    res = scan_kalman_full(q, k, v, r=r[None], a=a[None], qn=qn[None], S0=S0[None], P0=P0[None],
                           return_states=True)
    means, covs = _brute_force_posteriors(k[0], v[0], a, qn, r, S0, P0)
    np.testing.assert_allclose(res["S_hist"][0], means, rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(res["P_hist"][0], covs, rtol=1e-9, atol=1e-10)
    o_ref = np.einsum("tij,ti->tj", means, q[0])
    np.testing.assert_allclose(res["o"][0], o_ref, rtol=1e-9, atol=1e-10)


def test_kalman_covariance_symmetric_positive_definite_and_joseph_form():
    rng, q, k, v = _case(3, 60, 5, 2)
    L, dk = 60, 5
    a = 0.5 + 0.5 * rng.random(L)
    qn = 1e-3 * np.ones(L)
    r = 0.1 + rng.random(L)
    res = scan_kalman_full(q, k, v, r=r[None], a=a[None], qn=qn[None], return_states=True)
    P_prev = np.eye(dk)
    for t in range(L):
        P = res["P_hist"][0, t]
        assert np.abs(P - P.T).max() <= 1e-12 * np.abs(P).max()
        assert np.linalg.eigvalsh(P).min() > 0
        # Joseph form of the same update with the optimal gain: (I - g k^T) P- (I - g k^T)^T + r g g^T
        Pm = a[t] ** 2 * P_prev + qn[t] * np.eye(dk)
        kt = k[0, t]
        g = np.linalg.solve(np.linalg.inv(Pm) + np.outer(kt, kt) / r[t], kt / r[t])  # information-form gain
        J = np.eye(dk) - np.outer(g, kt)
        np.testing.assert_allclose(P, J @ Pm @ J.T + r[t] * np.outer(g, g), rtol=1e-9, atol=1e-12)
        P_prev = P


# ----------------------------------------------------------------------------- delta rule pins


def test_delta_is_kalman_with_isotropic_surrogate_covariance():
    """Kalman Delta Networks, Abstract; Memory by Design, Abstract.

    The delta rule is the Kalman update whose predictive covariance is replaced
    every token by an isotropic surrogate c_t I, with no covariance tracking.
    For unit keys, c_t / (c_t + r_t) = beta_t, i.e. c_t = beta_t r_t / (1 - beta_t).
    """
    rng, q, k, v = _case(4, 50, 6, 4)
    L, dk = 50, 6
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(L)))
    a = np.exp(-np.log1p(np.exp(rng.standard_normal(L) - 2.0)))  # exp(-softplus(x - 2))
    r = 0.1 + rng.random(L)
    res = scan_delta(q, k, v, beta[None], a=a[None], return_states=True)
    S = np.zeros((1, dk, 4))
    for t in range(L):
        c = beta[t] * r[t] / (1.0 - beta[t])
        S, _, g, e, _ = kalman_update(a[t] * S, c * np.eye(dk)[None], k[:, t], v[:, t], np.array([r[t]]))
        np.testing.assert_allclose(S[0], res["S_hist"][0, t], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(np.linalg.norm(g) * np.linalg.norm(e), res["m"][0, t], rtol=1e-10)


def test_delta_is_lms_gradient_step():
    """A Hippocampus for Linear Attention, section 3.3: the delta rule is the
    Widrow-Hoff / LMS rule, one gradient step of size beta_t on
    1/2 ||v_t - S^T k_t||^2 taken at the gated prediction a_t S_{t-1} (section 3.5).
    The gradient comes from autograd, not from the rule."""
    torch = pytest.importorskip("torch")
    rng, q, k, v = _case(5, 30, 5, 3)
    L = 30
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(L)))
    a = 0.4 + 0.6 * rng.random(L)
    res = scan_delta(q, k, v, beta[None], a=a[None], return_states=True)
    S = torch.zeros(5, 3, dtype=torch.float64)
    for t in range(L):
        Sp = (a[t] * S).detach().requires_grad_(True)
        kt = torch.from_numpy(k[0, t])
        vt = torch.from_numpy(v[0, t])
        loss = 0.5 * ((vt - Sp.T @ kt) ** 2).sum()
        (grad,) = torch.autograd.grad(loss, Sp)
        S = (Sp - beta[t] * grad).detach()
        np.testing.assert_allclose(S.numpy(), res["S_hist"][0, t], rtol=1e-11, atol=1e-13)


def test_delta_exact_recall_with_beta_one():
    # beta = 1 and a unit key: the write makes the memory return v_t at k_t (any gate)
    rng, q, k, v = _case(6, 25, 8, 3)
    a = 0.2 + 0.8 * rng.random(25)
    res = scan_delta(q, k, v, np.ones((1, 25)), a=a[None], return_states=True)
    for t in range(25):
        np.testing.assert_allclose(res["S_hist"][0, t].T @ k[0, t], v[0, t], rtol=1e-12, atol=1e-12)
    # orthonormal keys, a = 1: S = sum_i k_i v_i^T, so reading at k_0 returns v_0 from then on
    dk, L = 8, 6
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm[:L][None]
    vals = rng.standard_normal((1, L, 3))
    qs = np.repeat(keys[:, :1], L, axis=1)
    res = scan_delta(qs, keys, vals, np.ones((1, L)))
    np.testing.assert_allclose(res["S"][0], keys[0].T @ vals[0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(res["o"][0], np.repeat(vals[0, :1], L, axis=0), rtol=1e-12, atol=1e-12)


def test_delta_stability_bound_with_unit_keys():
    """A Hippocampus for Linear Attention, section 3.4: with ||k|| = 1 the operator
    I - beta k k^T has eigenvalues in [0, 1], so ||S_t||_2 <= a_t ||S_{t-1}||_2 + beta_t ||v_t||."""
    rng, q, k, v = _case(7, 200, 8, 4)
    beta = rng.random(200)
    a = rng.random(200)
    res = scan_delta(q, k, v, beta[None], a=a[None], return_states=True)
    prev = 0.0
    for t in range(200):
        ev = np.linalg.eigvalsh(np.eye(8) - beta[t] * np.outer(k[0, t], k[0, t]))
        assert ev.min() >= -1e-12 and ev.max() <= 1 + 1e-12
        n = np.linalg.norm(res["S_hist"][0, t], 2)
        assert n <= a[t] * prev + beta[t] * np.linalg.norm(v[0, t]) + 1e-12
        prev = n


def test_residual_reading_against_decayed_state():
    """Reading R1: the residual is against a_t S_{t-1}; the undecayed form agrees only when a = 1."""
    rng, q, k, v = _case(8, 20, 4, 3)
    beta = rng.random(20)
    a = 0.3 + 0.5 * rng.random(20)
    one = np.ones(20)
    r1 = scan_delta(q, k, v, beta[None], a=one[None])
    r2 = scan_delta(q, k, v, beta[None], a=one[None], residual="undecayed")
    np.testing.assert_allclose(r1["o"], r2["o"], rtol=1e-13, atol=1e-13)
    r3 = scan_delta(q, k, v, beta[None], a=a[None])
    r4 = scan_delta(q, k, v, beta[None], a=a[None], residual="undecayed")
    assert np.abs(r3["o"] - r4["o"]).max() > 1e-3


# ----------------------------------------------------------------------------- surprise


@pytest.mark.parametrize("variant", ["delta", "kalman_full", "kalman_diag", "kalman_iso"])
def test_surprise_is_frobenius_norm_of_the_write(variant):
    """A Hippocampus for Linear Attention, section 3.3, Eq. (6): m_t = ||Delta_t||_F,
    Delta_t = S_t - a_t S_{t-1} (the write, without the decay)."""
    rng, q, k, v = _case(9, 40, 6, 5)
    L = 40
    k = k * (0.5 + rng.random((1, L, 1)))  # non-unit keys: the norm of k is part of the write
    a = 0.5 + 0.5 * rng.random(L)
    r = 0.1 + rng.random(L)
    beta = rng.random(L)
    if variant == "delta":
        res = scan_delta(q, k, v, beta[None], a=a[None], return_states=True)
    elif variant == "kalman_full":
        res = scan_kalman_full(q, k, v, r=r[None], a=a[None], qn=1e-3, return_states=True)
    elif variant == "kalman_diag":
        res = scan_kalman_diag(q, k, v, r=r[None], a=a[None], qn=1e-3, return_states=True)
    else:
        res = scan_kalman_iso(q, k, v, r=r[None], a=a[None], qn=1e-3, return_states=True)
    S_prev = np.zeros((6, 5))
    for t in range(L):
        S_t = res["S_hist"][0, t]
        np.testing.assert_allclose(res["m"][0, t], np.linalg.norm(S_t - a[t] * S_prev, "fro"), rtol=1e-10,
                                   atol=1e-14)
        S_prev = S_t


# ----------------------------------------------------------------------------- diagonal variant


def test_diag_equals_full_on_one_hot_keys():
    """With one-hot keys and a diagonal P0 the exact posterior stays diagonal, so the
    diagonal projection loses nothing and the two variants coincide."""
    rng = np.random.default_rng(11)
    L, dk, dv = 40, 5, 3
    idx = rng.integers(0, dk, L)
    k = np.eye(dk)[idx][None]
    q = _unit_rows(rng.standard_normal((1, L, dk)))
    v = rng.standard_normal((1, L, dv))
    a = (0.5 + 0.5 * rng.random(L))[None]
    r = (0.1 + rng.random(L))[None]
    p0 = 0.5 + rng.random(dk)
    full = scan_kalman_full(q, k, v, r=r, a=a, qn=2e-2, P0=np.diag(p0)[None])
    diag = scan_kalman_diag(q, k, v, r=r, a=a, qn=2e-2, p0=p0[None])
    for key in ("o", "m", "S"):
        np.testing.assert_allclose(diag[key], full[key], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(diag["p"][0], np.diag(full["P"][0]), rtol=1e-12)
    assert np.abs(full["P"][0] - np.diag(np.diag(full["P"][0]))).max() < 1e-14


def test_diag_variances_closed_form_without_transition():
    """a = 1, Q = 0: each coordinate's precision accumulates k_i^2 / r, so
    p_L,i = 1 / (1/p0_i + sum_t k_ti^2 / r_t)."""
    rng, q, k, v = _case(12, 70, 7, 2)
    r = 0.1 + rng.random(70)
    p0 = 0.2 + rng.random(7)
    res = scan_kalman_diag(q, k, v, r=r[None], p0=p0[None])
    np.testing.assert_allclose(res["p"][0], 1.0 / (1.0 / p0 + (k[0] ** 2 / r[:, None]).sum(0)), rtol=1e-12)


def test_diag_mean_and_variances_are_conditioning_then_mean_field_projection():
    """Each step: the mean is exact Gaussian conditioning under the diagonal prior
    N(a S_{t-1}, diag(p-)) (explicit inverses), and the variances are the mean-field
    VI optimum, the reciprocals of the diagonal of the posterior precision."""
    rng, q, k, v = _case(13, 30, 5, 3)
    L = 30
    a = 0.5 + 0.5 * rng.random(L)
    r = 0.1 + rng.random(L)
    qn = 0.01
    res = scan_kalman_diag(q, k, v, r=r[None], a=a[None], qn=qn, return_states=True)
    S_prev, p_prev = np.zeros((5, 3)), np.ones(5)
    for t in range(L):
        p_pred = a[t] ** 2 * p_prev + qn
        kt = k[0, t]
        prior_prec = np.diag(1.0 / p_pred)
        post_prec = prior_prec + np.outer(kt, kt) / r[t]
        post_cov = np.linalg.inv(post_prec)
        mean = post_cov @ (prior_prec @ (a[t] * S_prev) + np.outer(kt, v[0, t]) / r[t])
        np.testing.assert_allclose(res["S_hist"][0, t], mean, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(res["p_hist"][0, t], 1.0 / np.diag(np.linalg.inv(post_cov)), rtol=1e-10)
        S_prev, p_prev = res["S_hist"][0, t], res["p_hist"][0, t]


def test_diag_variances_minimise_reverse_kl():
    """Online mean-field VI (Kalman Delta Networks, Abstract) minimises KL(q || posterior)
    over diagonal Gaussians q; minimise it numerically and compare."""
    scipy_opt = pytest.importorskip("scipy.optimize")
    rng = np.random.default_rng(14)
    dk = 4
    p_pred = 0.3 + rng.random(dk)
    kt = _unit_rows(rng.standard_normal(dk))
    r = 0.4
    post_cov = np.diag(p_pred) - np.outer(p_pred * kt, p_pred * kt) / (p_pred @ (kt * kt) + r)
    prec = np.linalg.inv(post_cov)

    def kl(logvar):  # KL(N(mu, diag(exp logvar)) || N(mu, post_cov)), up to constants
        var = np.exp(logvar)
        return 0.5 * (np.sum(np.diag(prec) * var) - np.sum(logvar))

    opt = scipy_opt.minimize(kl, np.zeros(dk), method="BFGS", options={"gtol": 1e-12})
    S_pred = np.zeros((1, dk, 1))
    res = scan_kalman_diag(np.zeros((1, 1, dk)), kt[None, None], np.zeros((1, 1, 1)), r=np.array([[r]]),
                           p0=p_pred[None])
    np.testing.assert_allclose(res["p"][0], np.exp(opt.x), rtol=1e-6)
    assert S_pred.shape == (1, dk, 1)


# ----------------------------------------------------------------------------- isotropic variant
# Kalman Delta Networks, Abstract: Isotropic KDN keeps a single uncertainty scalar per head (reading R12).


def test_iso_equals_full_kalman_in_one_dimension():
    """With d_k = 1 every covariance is a scalar, so the isotropic projection is exact and
    the variant is the full Kalman filter (and the diagonal one)."""
    rng = np.random.default_rng(21)
    L, dv, n = 50, 4, 3
    q = rng.standard_normal((n, L, 1))
    k = rng.standard_normal((n, L, 1))
    v = rng.standard_normal((n, L, dv))
    a = 0.4 + 0.6 * rng.random((n, L))
    r = 0.1 + rng.random((n, L))
    c0 = 0.3 + rng.random(n)
    iso = scan_kalman_iso(q, k, v, r=r, a=a, qn=3e-2, c0=c0)
    full = scan_kalman_full(q, k, v, r=r, a=a, qn=3e-2, P0=c0[:, None, None])
    for key in ("o", "m", "S"):
        np.testing.assert_allclose(iso[key], full[key], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(iso["c"], full["P"][:, 0, 0], rtol=1e-12)


def test_iso_variance_closed_form_without_transition():
    """a = 1, Q = 0: the trace of the precision grows by ||k_t||^2 / r_t per token, so
    d_k / c_L = d_k / c0 + sum_t ||k_t||^2 / r_t (non-unit keys)."""
    rng, q, k, v = _case(22, 60, 6, 3)
    k = k * (0.3 + rng.random((1, 60, 1)))
    r = 0.1 + rng.random(60)
    c0 = 0.7
    res = scan_kalman_iso(q, k, v, r=r[None], c0=np.array([c0]))
    dk = 6
    np.testing.assert_allclose(res["c"][0], dk / (dk / c0 + ((k[0] ** 2).sum(-1) / r).sum()), rtol=1e-12)


def test_iso_mean_and_variance_are_conditioning_then_isotropic_projection():
    """Each step: the mean is exact Gaussian conditioning under the isotropic prior
    N(a S_{t-1}, c^- I) (explicit inverses), and the variance is d_k over the trace of the
    posterior precision."""
    rng, q, k, v = _case(23, 30, 5, 3)
    L = 30
    k = k * (0.5 + rng.random((1, L, 1)))
    a = 0.5 + 0.5 * rng.random(L)
    r = 0.1 + rng.random(L)
    qn = 0.02
    res = scan_kalman_iso(q, k, v, r=r[None], a=a[None], qn=qn, return_states=True)
    S_prev, c_prev = np.zeros((5, 3)), 1.0
    for t in range(L):
        c_pred = a[t] ** 2 * c_prev + qn
        kt = k[0, t]
        prior_prec = np.eye(5) / c_pred
        post_prec = prior_prec + np.outer(kt, kt) / r[t]
        post_cov = np.linalg.inv(post_prec)
        mean = post_cov @ (prior_prec @ (a[t] * S_prev) + np.outer(kt, v[0, t]) / r[t])
        np.testing.assert_allclose(res["S_hist"][0, t], mean, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(res["c_hist"][0, t], 5.0 / np.trace(post_prec), rtol=1e-12)
        S_prev, c_prev = res["S_hist"][0, t], res["c_hist"][0, t]


def test_iso_variance_minimises_reverse_kl():
    """The isotropic projection minimises KL(N(mu, c I) || posterior) over c; minimise it
    numerically and compare."""
    scipy_opt = pytest.importorskip("scipy.optimize")
    rng = np.random.default_rng(24)
    dk = 4
    c_pred = 0.8
    kt = rng.standard_normal(dk)
    r = 0.3
    prec = np.eye(dk) / c_pred + np.outer(kt, kt) / r

    def kl(logc):  # KL(N(mu, exp(logc) I) || N(mu, prec^-1)), up to constants
        return 0.5 * (np.exp(logc[0]) * np.trace(prec) - dk * logc[0])

    opt = scipy_opt.minimize(kl, np.zeros(1), method="BFGS", options={"gtol": 1e-12})
    res = scan_kalman_iso(np.zeros((1, 1, dk)), kt[None, None], np.zeros((1, 1, 1)), r=np.array([[r]]),
                          c0=np.array([c_pred]))
    np.testing.assert_allclose(res["c"][0], np.exp(opt.x[0]), rtol=1e-6)


def test_iso_is_the_delta_rule_with_a_variance_driven_beta():
    """The isotropic gain is c^- k / (c^- ||k||^2 + r): the delta rule's write with
    beta_t = c^-_t / (c^-_t ||k_t||^2 + r_t)."""
    rng, q, k, v = _case(25, 40, 6, 4)
    L = 40
    k = k * (0.5 + rng.random((1, L, 1)))
    a = 0.5 + 0.5 * rng.random(L)
    r = 0.1 + rng.random(L)
    qn = 1e-2
    iso = scan_kalman_iso(q, k, v, r=r[None], a=a[None], qn=qn, return_states=True)
    c_prev = np.concatenate([[1.0], iso["c_hist"][0, :-1]])
    c_pred = a * a * c_prev + qn
    beta = c_pred / (c_pred * (k[0] ** 2).sum(-1) + r)
    delta = scan_delta(q, k, v, beta[None], a=a[None])
    for key in ("o", "m", "S"):
        np.testing.assert_allclose(iso[key], delta[key], rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------------------------- decode


@pytest.mark.parametrize("variant", ["delta", "kalman_diag", "kalman_iso"])
def test_n_decode_steps_equal_a_scan(variant):
    rng, q, k, v = _case(15, 12, 6, 4, heads=(2, 3))
    beta = rng.random((2, 3, 12))
    a = 0.5 + 0.5 * rng.random((2, 3, 12))
    r = 0.1 + rng.random((2, 3, 12))
    if variant == "delta":
        ref = scan_delta(q, k, v, beta, a=a)
    elif variant == "kalman_diag":
        ref = scan_kalman_diag(q, k, v, r=r, a=a, qn=1e-3)
    else:
        ref = scan_kalman_iso(q, k, v, r=r, a=a, qn=1e-3)
    S = np.zeros((2, 3, 6, 4))
    p = np.ones((2, 3)) if variant == "kalman_iso" else np.ones((2, 3, 6))
    for t in range(12):
        st = decode_step(variant, q[..., t, :], k[..., t, :], v[..., t, :], S, beta=beta[..., t], a=a[..., t],
                         r=r[..., t], qn=1e-3, p=p)
        np.testing.assert_allclose(st["o"], ref["o"][..., t, :], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(st["m"], ref["m"][..., t], rtol=1e-12, atol=1e-13)
        S = st["S"]
        p = st.get("p", p)
    np.testing.assert_allclose(S, ref["S"], rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------------------------- hand-derived values


def _frac(x):
    return float(Fraction(x))


def test_golden_hand_derived_examples():
    with open(os.path.join(GOLDEN, "hand_derived_steps.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        inp = {name: np.array([[[_frac(x) for x in row] for row in c["inputs"][name]]])
               for name in ("q", "k", "v")}
        sc = {name: np.array([[_frac(x) for x in c["inputs"][name]]]) for name in c["inputs"]
              if name in ("beta", "a", "r", "qn")}
        if c["variant"] == "delta":
            res = scan_delta(inp["q"], inp["k"], inp["v"], sc["beta"], a=sc.get("a"))
        elif c["variant"] == "kalman_full":
            S0 = np.array([[[_frac(x) for x in row] for row in c["inputs"]["S0"]]]) if "S0" in c["inputs"] else None
            P0 = np.array([[[_frac(x) for x in row] for row in c["inputs"]["P0"]]])
            res = scan_kalman_full(inp["q"], inp["k"], inp["v"], r=sc["r"], a=sc.get("a"), qn=sc.get("qn"),
                                   S0=S0, P0=P0)
        else:
            p0 = np.array([[_frac(x) for x in c["inputs"]["p0"]]])
            res = scan_kalman_diag(inp["q"], inp["k"], inp["v"], r=sc["r"], a=sc.get("a"), qn=sc.get("qn"), p0=p0)
        exp = c["expected"]
        np.testing.assert_allclose(res["o"][0], [[_frac(x) for x in row] for row in exp["o"]], rtol=1e-13,
                                   atol=1e-15, err_msg=c["name"])
        np.testing.assert_allclose(res["m"][0], [eval_m(x) for x in exp["m"]], rtol=1e-13, atol=1e-15,
                                   err_msg=c["name"])
        np.testing.assert_allclose(res["S"][0], [[_frac(x) for x in row] for row in exp["S"]], rtol=1e-13,
                                   atol=1e-15, err_msg=c["name"])
        if "P" in exp:
            np.testing.assert_allclose(res["P"][0], [[_frac(x) for x in row] for row in exp["P"]], rtol=1e-13)
        if "p" in exp:
            np.testing.assert_allclose(res["p"][0], [_frac(x) for x in exp["p"]], rtol=1e-13)


def eval_m(x):
    """m values are stored as 'num' or 'sqrt(num)/den' strings of exact fractions."""
    if x.startswith("sqrt("):
        inner, den = x[5:].split(")/")
        return float(np.sqrt(_frac(inner)) / _frac(den))
    return _frac(x)
