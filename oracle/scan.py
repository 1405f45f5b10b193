"""Float64 CPU oracle for the gain-weighted residual memory scan.

TEST INFRASTRUCTURE ONLY.  The product package (``delta_rule_recurrent_scan_b200``)
never imports, links or runs anything in ``oracle/``; only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference arm do.
This module imports nothing from the product either: the two sides share no code.

It is plain, slow and written to be checked against the pages by eye: NumPy in
float64, one token at a time, vectorised only over the independent heads
(b, h).  Inputs are upcast exactly to float64 (bf16 and fp32 values are exact
in float64).

Per head the memory is a matrix S (d_k x d_v) read as o_t = S_t^T q_t.  Every
variant writes it with a gain-weighted residual

    S_t = a_t S_{t-1} + g_t e_t^T,    e_t = v_t - (a_t S_{t-1})^T k_t,

and differs only in the gain g_t:

* gated delta rule     g_t = beta_t k_t
      A Hippocampus for Linear Attention, section 3.3, Eq. (5) (rank-1 write
      Delta_t = beta_t k_t e_t^T) and section 3.5 "Instantiation (GDN)" (gate
      alpha_t in (0, 1], prediction alpha_t k^T S_{t-1}, residual against it).
* full-covariance Kalman / RLS   g_t = P^- k_t / (k_t^T P^- k_t + r_t)
      Kalman Delta Networks, Abstract (linear-Gaussian state-space memory,
      Kalman gain, Riccati recursion, transition propagates state and
      uncertainty); Memory by Design, Abstract (exact Bayesian filtering of
      mean and covariance); DeltaNet-PC, "How it works", Eq. (5)-(7) (ridge
      energy and its recursive least-squares minimiser).
* diagonal-covariance Kalman    g_t = p^- * k_t / (sum_i p^-_i k_ti^2 + r_t)
      Kalman Delta Networks, Abstract (each one-step posterior projected onto
      diagonal Gaussians by online mean-field variational inference).

and every variant emits the surprise score m_t = ||g_t e_t^T||_F =
||g_t|| ||e_t|| (A Hippocampus for Linear Attention, section 3.3, Eq. (6)).

Readings where the pages leave a step open (the same list is kept with the
design notes of the repository):

R1  The residual is taken against the decayed (predicted) state a_t S_{t-1}
    (section 3.5 of the HOLA page; standard predict-then-update).  The
    undecayed form v_t - S_{t-1}^T k_t is available as ``residual="undecayed"``
    for the delta rule only, to document the difference; the two agree at a=1.
R2  Kalman order per token: propagate (P^- = a_t^2 P + Qn_t I, S^- = a_t S),
    then update with token t.  P_0 is the posterior before token 1 and the
    returned P_L is the posterior after token L, not propagated further.
R3  Diagonal variant: the mean is the exact posterior mean under the diagonal
    prior (so the gain above), and the variances are those of the mean-field
    VI optimum, KL(q || posterior) over diagonal Gaussians, which keeps the
    inverse of the diagonal of the posterior precision:
    p_i = 1 / (1/p^-_i + k_i^2 / r) = p^-_i r / (r + p^-_i k_i^2).
    Per coordinate this composed with p -> a^2 p + Qn is a Moebius map, which is
    what the KDN abstract says of its scan-compatible uncertainty recurrences.
R4  Surprise for every variant is the Frobenius norm of the write, excluding
    the decay: m_t = ||g_t|| ||e_t||.  For the delta rule that is
    beta_t ||k_t|| ||e_t|| (equal to beta_t ||e_t|| when ||k_t|| = 1).
R5  The read uses the post-update state and no 1/sqrt(d) scale.
R6  Orientation: S is d_k x d_v and the read is S^T q (HOLA and the GDN gate
    formula); the DeltaNet-PC page writes the transpose, S k.
R12 Isotropic variant (one uncertainty scalar c per head; the KDN abstract
    gives no formula): propagate c^- = a_t^2 c + Qn_t; the mean is the exact
    posterior mean under the prior c^- I, so g_t = c^- k_t / (c^- ||k_t||^2 + r_t);
    the variance is the isotropic mean-field optimum, KL(q || posterior) over
    N(mu, c I), c = d_k / tr(posterior precision) = d_k c^- r / (d_k r + c^- ||k||^2).
    Composed with the propagation this is again a Moebius map of c, and the
    write is the delta rule's with beta_t = c^- / (c^- ||k_t||^2 + r_t).

Pins (tests/test_oracle_pins.py): the ridge closed form for every prefix,
brute-force joint-Gaussian conditioning on tiny inputs, the isotropic-surrogate
reduction of Kalman to the delta rule, the LMS / gradient-step reading of the
delta rule (autograd), exact recall with beta = 1, m_t = ||S_t - a_t S_{t-1}||_F,
P symmetric positive definite and equal to the Joseph form, the diagonal
closed form at a = 1, Q = 0, the diagonal = full identity on one-hot keys, the
VI optimality of the diagonal variances (explicit inverse and a numerical KL
minimisation), and hand-derived worked values in tests/golden/.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "scan_delta",
    "scan_kalman_full",
    "scan_kalman_diag",
    "decode_step",
    "kalman_update",
    "diag_update",
    "scan_kalman_iso",
    "iso_update",
]


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def _per_token(x, n_heads, L, default):
    """Return a (n_heads, L) float64 array from None, a scalar or a [.., L] array."""
    if x is None:
        return np.full((n_heads, L), float(default))
    x = _f64(x)
    if x.ndim == 0:
        return np.full((n_heads, L), float(x))
    return x.reshape(n_heads, L)


def _flatten_inputs(q, k, v):
    q, k, v = _f64(q), _f64(k), _f64(v)
    lead = k.shape[:-2]
    L, dk = k.shape[-2:]
    dv = v.shape[-1]
    n = int(np.prod(lead)) if lead else 1
    return lead, n, L, dk, dv, q.reshape(n, L, dk), k.reshape(n, L, dk), v.reshape(n, L, dv)


def _read(S, x):
    """S^T x for a stack of heads: S (n, dk, dv), x (n, dk) -> (n, dv)."""
    return np.einsum("nij,ni->nj", S, x)


# --------------------------------------------------------------------------- delta rule


def scan_delta(q, k, v, beta, a=None, S0=None, residual="predicted", return_states=False):
    """Gated delta rule, token by token.

    A Hippocampus for Linear Attention, section 3.3, Eq. (5): the token's whole
    effect on the memory is the rank-1 write Delta_t = beta_t k_t e_t^T; section
    3.5: the GDN gate alpha_t (here ``a``) multiplies S_{t-1} and the residual is
    taken against that prediction, e_t = v_t - alpha_t S_{t-1}^T k_t.  Eq. (6):
    m_t = ||Delta_t||_F = beta_t ||k_t|| ||e_t||.

    Shapes: q, k [..., L, d_k]; v [..., L, d_v]; beta, a [..., L]; S0 [..., d_k, d_v].
    ``a=None`` is the plain (ungated) delta rule, a_t = 1.  Returns a dict with
    o [..., L, d_v], m [..., L], S [..., d_k, d_v] (final state) and, with
    ``return_states``, S_hist [..., L, d_k, d_v] (the state after each token).
    """
    if residual not in ("predicted", "undecayed"):
        raise ValueError("residual must be 'predicted' or 'undecayed'")
    lead, n, L, dk, dv, q, k, v = _flatten_inputs(q, k, v)
    beta = _per_token(beta, n, L, 0.0)
    a = _per_token(a, n, L, 1.0)
    S = np.zeros((n, dk, dv)) if S0 is None else _f64(S0).reshape(n, dk, dv).copy()
    o = np.zeros((n, L, dv))
    m = np.zeros((n, L))
    hist = np.zeros((n, L, dk, dv)) if return_states else None
    for t in range(L):
        kt, vt = k[:, t], v[:, t]
        S_pred = a[:, t, None, None] * S
        base = S_pred if residual == "predicted" else S
        e = vt - _read(base, kt)
        write = beta[:, t, None, None] * kt[:, :, None] * e[:, None, :]
        S = S_pred + write
        o[:, t] = _read(S, q[:, t])
        m[:, t] = beta[:, t] * np.linalg.norm(kt, axis=-1) * np.linalg.norm(e, axis=-1)
        if hist is not None:
            hist[:, t] = S
    out = {
        "o": o.reshape(*lead, L, dv),
        "m": m.reshape(*lead, L),
        "S": S.reshape(*lead, dk, dv),
    }
    if hist is not None:
        out["S_hist"] = hist.reshape(*lead, L, dk, dv)
    return out


# --------------------------------------------------------------------------- full Kalman


def kalman_update(S_pred, P_pred, k, v, r):
    """Measurement update of the linear-Gaussian memory for one token.

    Kalman Delta Networks, Abstract: the Kalman gain weights the residual write
    by the accumulated evidence (P) and the observation reliability (r).
    DeltaNet-PC, Eq. (7): the recursive least-squares form of the same update.

    S_pred (n, dk, dv), P_pred (n, dk, dk), k (n, dk), v (n, dv), r (n,).
    Returns (S, P, g, e, s): posterior mean and covariance, gain, innovation,
    innovation variance.
    """
    e = v - _read(S_pred, k)
    Pk = np.einsum("nij,nj->ni", P_pred, k)
    s = np.einsum("ni,ni->n", k, Pk) + r
    g = Pk / s[:, None]
    S = S_pred + g[:, :, None] * e[:, None, :]
    # P <- P - g k^T P, written in its symmetric form P - s g g^T (equal in exact arithmetic)
    P = P_pred - s[:, None, None] * g[:, :, None] * g[:, None, :]
    return S, P, g, e, s


def scan_kalman_full(q, k, v, r, a=None, qn=None, S0=None, P0=None, return_states=False):
    """Full-covariance Kalman / RLS memory, token by token (reading R2: predict, then update).

    Per token: S^- = a_t S, P^- = a_t^2 P + Qn_t I (Kalman Delta Networks,
    Abstract: the transition propagates both the memory and its uncertainty),
    then ``kalman_update``.  o_t = S_t^T q_t, m_t = ||g_t|| ||e_t||.

    r [..., L] (observation-noise variance), a [..., L] or None (=1),
    qn [..., L], a scalar or None (=0) (process noise Q_t = qn_t I),
    S0 [..., d_k, d_v] or None (=0), P0 [..., d_k, d_k] or None (=I).
    Returns o, m, S, P and, with ``return_states``, S_hist and P_hist.
    """
    lead, n, L, dk, dv, q, k, v = _flatten_inputs(q, k, v)
    r = _per_token(r, n, L, 1.0)
    a = _per_token(a, n, L, 1.0)
    qn = _per_token(qn, n, L, 0.0)
    S = np.zeros((n, dk, dv)) if S0 is None else _f64(S0).reshape(n, dk, dv).copy()
    P = np.broadcast_to(np.eye(dk), (n, dk, dk)).copy() if P0 is None else _f64(P0).reshape(n, dk, dk).copy()
    eye = np.eye(dk)
    o = np.zeros((n, L, dv))
    m = np.zeros((n, L))
    S_hist = np.zeros((n, L, dk, dv)) if return_states else None
    P_hist = np.zeros((n, L, dk, dk)) if return_states else None
    for t in range(L):
        at = a[:, t, None, None]
        S_pred = at * S
        P_pred = at * at * P + qn[:, t, None, None] * eye
        S, P, g, e, _ = kalman_update(S_pred, P_pred, k[:, t], v[:, t], r[:, t])
        o[:, t] = _read(S, q[:, t])
        m[:, t] = np.linalg.norm(g, axis=-1) * np.linalg.norm(e, axis=-1)
        if return_states:
            S_hist[:, t] = S
            P_hist[:, t] = P
    out = {
        "o": o.reshape(*lead, L, dv),
        "m": m.reshape(*lead, L),
        "S": S.reshape(*lead, dk, dv),
        "P": P.reshape(*lead, dk, dk),
    }
    if return_states:
        out["S_hist"] = S_hist.reshape(*lead, L, dk, dv)
        out["P_hist"] = P_hist.reshape(*lead, L, dk, dk)
    return out


# --------------------------------------------------------------------------- diagonal Kalman


def diag_update(S_pred, p_pred, k, v, r):
    """Measurement update with a diagonal prior covariance diag(p_pred) (reading R3).

    Kalman Delta Networks, Abstract: Diagonal KDN projects each one-step
    posterior onto the diagonal Gaussian family through online mean-field
    variational inference.  The posterior mean is the exact conditional mean
    under the diagonal prior; the projected variances are the reciprocals of the
    diagonal of the posterior precision, diag(1/p_pred) + k k^T / r.

    Returns (S, p, g, e, s).
    """
    e = v - _read(S_pred, k)
    s = np.einsum("ni,ni->n", p_pred, k * k) + r
    g = p_pred * k / s[:, None]
    S = S_pred + g[:, :, None] * e[:, None, :]
    p = p_pred * r[:, None] / (r[:, None] + p_pred * k * k)
    return S, p, g, e, s


def scan_kalman_diag(q, k, v, r, a=None, qn=None, S0=None, p0=None, return_states=False):
    """Diagonal-covariance Kalman memory, token by token.

    Per token: S^- = a_t S, p^- = a_t^2 p + Qn_t, then ``diag_update``.
    p0 [..., d_k] or None (=1).  Returns o, m, S, p and, with
    ``return_states``, S_hist and p_hist.
    """
    lead, n, L, dk, dv, q, k, v = _flatten_inputs(q, k, v)
    r = _per_token(r, n, L, 1.0)
    a = _per_token(a, n, L, 1.0)
    qn = _per_token(qn, n, L, 0.0)
    S = np.zeros((n, dk, dv)) if S0 is None else _f64(S0).reshape(n, dk, dv).copy()
    p = np.ones((n, dk)) if p0 is None else _f64(p0).reshape(n, dk).copy()
    o = np.zeros((n, L, dv))
    m = np.zeros((n, L))
    S_hist = np.zeros((n, L, dk, dv)) if return_states else None
    p_hist = np.zeros((n, L, dk)) if return_states else None
    for t in range(L):
        at = a[:, t]
        S_pred = at[:, None, None] * S
        p_pred = (at * at)[:, None] * p + qn[:, t, None]
        S, p, g, e, _ = diag_update(S_pred, p_pred, k[:, t], v[:, t], r[:, t])
        o[:, t] = _read(S, q[:, t])
        m[:, t] = np.linalg.norm(g, axis=-1) * np.linalg.norm(e, axis=-1)
        if return_states:
            S_hist[:, t] = S
            p_hist[:, t] = p
    out = {
        "o": o.reshape(*lead, L, dv),
        "m": m.reshape(*lead, L),
        "S": S.reshape(*lead, dk, dv),
        "p": p.reshape(*lead, dk),
    }
    if return_states:
        out["S_hist"] = S_hist.reshape(*lead, L, dk, dv)
        out["p_hist"] = p_hist.reshape(*lead, L, dk)
    return out


# --------------------------------------------------------------------------- isotropic Kalman


def iso_update(S_pred, c_pred, k, v, r):
    """Measurement update with an isotropic prior covariance c_pred I (reading R12).

    Kalman Delta Networks, Abstract: Isotropic KDN uses an isotropic
    approximation with a single uncertainty scalar per head.  The posterior
    mean is the exact conditional mean under the prior c_pred I; the projected
    variance is d_k over the trace of the posterior precision
    I / c_pred + k k^T / r, written without dividing by c_pred.

    Returns (S, c, g, e, s).
    """
    dk = k.shape[-1]
    e = v - _read(S_pred, k)
    kk = np.einsum("ni,ni->n", k, k)
    s = c_pred * kk + r
    g = (c_pred / s)[:, None] * k
    S = S_pred + g[:, :, None] * e[:, None, :]
    c = dk * c_pred * r / (dk * r + c_pred * kk)
    return S, c, g, e, s


def scan_kalman_iso(q, k, v, r, a=None, qn=None, S0=None, c0=None, return_states=False):
    """Isotropic-covariance Kalman memory, token by token.

    Per token: S^- = a_t S, c^- = a_t^2 c + Qn_t, then ``iso_update``.
    c0 [...] or None (=1).  Returns o, m, S, c and, with ``return_states``,
    S_hist and c_hist.
    """
    lead, n, L, dk, dv, q, k, v = _flatten_inputs(q, k, v)
    r = _per_token(r, n, L, 1.0)
    a = _per_token(a, n, L, 1.0)
    qn = _per_token(qn, n, L, 0.0)
    S = np.zeros((n, dk, dv)) if S0 is None else _f64(S0).reshape(n, dk, dv).copy()
    c = np.ones(n) if c0 is None else _f64(c0).reshape(n).copy()
    o = np.zeros((n, L, dv))
    m = np.zeros((n, L))
    S_hist = np.zeros((n, L, dk, dv)) if return_states else None
    c_hist = np.zeros((n, L)) if return_states else None
    for t in range(L):
        at = a[:, t]
        S_pred = at[:, None, None] * S
        c_pred = at * at * c + qn[:, t]
        S, c, g, e, _ = iso_update(S_pred, c_pred, k[:, t], v[:, t], r[:, t])
        o[:, t] = _read(S, q[:, t])
        m[:, t] = np.linalg.norm(g, axis=-1) * np.linalg.norm(e, axis=-1)
        if return_states:
            S_hist[:, t] = S
            c_hist[:, t] = c
    out = {
        "o": o.reshape(*lead, L, dv),
        "m": m.reshape(*lead, L),
        "S": S.reshape(*lead, dk, dv),
        "c": c.reshape(lead),
    }
    if return_states:
        out["S_hist"] = S_hist.reshape(*lead, L, dk, dv)
        out["c_hist"] = c_hist.reshape(*lead, L)
    return out


# --------------------------------------------------------------------------- decode


def decode_step(variant, q, k, v, S, beta=None, a=None, r=None, qn=None, p=None):
    """One recurrent token against a resident state: the scan above with L = 1.

    Kalman Delta Networks, Abstract (constant-memory decoding with a fixed-size
    recurrent memory).  q, k [..., d_k]; v [..., d_v]; beta, a, r [...] or None;
    qn a scalar, [...] or None; S [..., d_k, d_v]; p [..., d_k] (diagonal) or the
    uncertainty scalar [...] (isotropic).  ``variant`` is "delta", "kalman_diag" or
    "kalman_iso".  Returns o [..., d_v], m [...],
    S and (diagonal) p after the token.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    lead = k.shape[:-1]

    def tok(x):
        return None if x is None else _f64(x)[..., None]

    def tokvec(x):
        return x[..., None, :]

    if variant == "delta":
        res = scan_delta(tokvec(q), tokvec(k), tokvec(v), tok(beta), a=tok(a), S0=S)
        return {"o": res["o"][..., 0, :], "m": res["m"][..., 0], "S": res["S"]}
    if variant == "kalman_diag":
        qn_t = None if qn is None else (np.broadcast_to(_f64(qn), lead)[..., None])
        res = scan_kalman_diag(tokvec(q), tokvec(k), tokvec(v), tok(r), a=tok(a), qn=qn_t, S0=S, p0=p)
        return {"o": res["o"][..., 0, :], "m": res["m"][..., 0], "S": res["S"], "p": res["p"]}
    if variant == "kalman_iso":  # p is the uncertainty scalar c [...]
        qn_t = None if qn is None else (np.broadcast_to(_f64(qn), lead)[..., None])
        res = scan_kalman_iso(tokvec(q), tokvec(k), tokvec(v), tok(r), a=tok(a), qn=qn_t, S0=S, c0=p)
        return {"o": res["o"][..., 0, :], "m": res["m"][..., 0], "S": res["S"], "p": res["c"]}
    raise ValueError(f"unknown decode variant {variant!r}")
