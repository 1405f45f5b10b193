"""Float64 reverse-mode derivatives of the gated delta rule and diagonal-Kalman scans (the backward pass).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: nothing in the product package imports it.

The pages train the layers these scans come from (A Hippocampus for Linear Attention, section 4: models
pretrained at 340M to 1.3B parameters; Kalman Delta Networks, Abstract: the KDN layers are trained
end to end), but print no backward pass.  This is the plainest one: the adjoint of the token-by-token
recurrence of ``oracle.scan.scan_delta``, written out by the chain rule and run backwards in time.

Forward, per head (section 3.3 Eq. (5)-(6) and section 3.5 of the HOLA page):

    e_t = v_t - a_t S_{t-1}^T k_t,   S_t = a_t S_{t-1} + beta_t k_t e_t^T,
    o_t = S_t^T q_t,                 m_t = beta_t ||k_t|| ||e_t||.

For a scalar loss with upstream gradients dO_t = dLoss/do_t, dm_t = dLoss/dm_t and dS_L = dLoss/dS_L, let
G_t = dLoss/dS_t (everything that reaches S_t, including through later tokens).  Backwards from t = L:

    G_t     += q_t dO_t^T                         (the read o_t = S_t^T q_t)
    dq_t     = S_t dO_t
    de_t     = beta_t G_t^T k_t + dm_t beta_t ||k_t|| e_t / ||e_t||
    dbeta_t  = k_t^T G_t e_t + dm_t ||k_t|| ||e_t||
    dk_t     = beta_t G_t e_t + dm_t beta_t ||e_t|| k_t / ||k_t||  -  a_t S_{t-1} de_t
    dv_t     = de_t
    da_t     = <G_t, S_{t-1}>  -  k_t^T S_{t-1} de_t
    G_{t-1}  = a_t G_t  -  a_t k_t de_t^T

and dS_0 = G_0.  The states S_{t-1} are kept from a forward pass (this is the oracle: memory is no object).
A zero residual or a zero key contributes no surprise gradient (the norm is not differentiable there; the
one-sided choice 0 is taken).

The diagonal-Kalman variant (Kalman Delta Networks, Abstract; the mean-field reading R3 of
``oracle.scan``) adds the variance vector p to the state.  Per token

    p^- = a_t^2 p + Qn_t,  s_t = sum_i p^-_i k_ti^2 + r_t,  g_t = p^- o k_t / s_t,
    p   = p^- r_t / (r_t + p^- o k_t^2),

and the write is S_t = a_t S_{t-1} + g_t e_t^T with m_t = ||g_t|| ||e_t||.  Its backward carries the
adjoint Pb = dLoss/dp next to G: from g, dp^- = dg o k / s, ds = -(dg . g) / s, dk += dg o p^- / s; from
the projection p = p^- r / den (den = r + p^- k^2), dp^- += Pb r^2 / den^2, dr += sum Pb (p^- k)^2 / den^2,
dk -= 2 Pb (p^-)^2 r k / den^2; from s, dp^- += ds k^2, dk += 2 ds p^- k, dr += ds; and through the
propagation Pb_{t-1} = a_t^2 dp^-, da_t += 2 a_t (dp^- . p_{t-1}), dQn_t = sum dp^-.

The isotropic variant (reading R12) carries one scalar c: c^- = a^2 c + Qn, s = c^- ||k||^2 + r,
g = (c^- / s) k, c = d_k c^- r / (d_k r + c^- ||k||^2); and the full-covariance variant carries P:
P^- = a^2 P + Qn I, u = P^- k, s = k^T u + r, g = u / s, P = P^- - u u^T / s (the symmetric form the forward
oracle uses).  Their backwards follow the same pattern: the memory part gives dg, which runs back through
the gain and the uncertainty update, and the uncertainty adjoint is carried to the previous token.
"""

from __future__ import annotations

import numpy as np

from .scan import _f64, _flatten_inputs, _per_token, _read

__all__ = ["scan_delta_backward", "scan_kalman_diag_backward", "scan_kalman_iso_backward",
           "scan_kalman_full_backward"]


def scan_delta_backward(q, k, v, beta, dO, a=None, S0=None, dm=None, dS_L=None):
    """Gradients of the gated delta rule scan.

    Shapes as ``oracle.scan.scan_delta``: q, k [..., L, d_k]; v [..., L, d_v]; beta, a [..., L];
    S0 [..., d_k, d_v] (None = 0); upstream dO [..., L, d_v], dm [..., L] or None, dS_L [..., d_k, d_v] or
    None.  Returns a dict of float64 arrays dq, dk, dv, dbeta, da (da is returned even for a=None, as the
    gradient at a_t = 1) and dS0, each with its input's shape.
    """
    lead, n, L, dk, dv, q, k, v = _flatten_inputs(q, k, v)
    beta = _per_token(beta, n, L, 0.0)
    a = _per_token(a, n, L, 1.0)
    dO = _f64(dO).reshape(n, L, dv)
    dm = _per_token(dm, n, L, 0.0)
    S = np.zeros((n, dk, dv)) if S0 is None else _f64(S0).reshape(n, dk, dv).copy()

    # forward, keeping every state and residual
    states = np.zeros((n, L + 1, dk, dv))
    states[:, 0] = S
    res = np.zeros((n, L, dv))
    for t in range(L):
        kt = k[:, t]
        S_pred = a[:, t, None, None] * S
        e = v[:, t] - _read(S_pred, kt)
        S = S_pred + beta[:, t, None, None] * kt[:, :, None] * e[:, None, :]
        states[:, t + 1] = S
        res[:, t] = e

    # backward
    G = np.zeros((n, dk, dv)) if dS_L is None else _f64(dS_L).reshape(n, dk, dv).copy()
    dq = np.zeros((n, L, dk))
    dkk = np.zeros((n, L, dk))
    dvv = np.zeros((n, L, dv))
    dbeta = np.zeros((n, L))
    da = np.zeros((n, L))
    for t in range(L - 1, -1, -1):
        kt, qt, e = k[:, t], q[:, t], res[:, t]
        S_t, S_prev = states[:, t + 1], states[:, t]
        bt, at = beta[:, t], a[:, t]
        G = G + qt[:, :, None] * dO[:, t, None, :]
        dq[:, t] = np.einsum("nij,nj->ni", S_t, dO[:, t])
        kn = np.linalg.norm(kt, axis=-1)
        en = np.linalg.norm(e, axis=-1)
        e_dir = np.where(en[:, None] > 0, e / np.where(en > 0, en, 1.0)[:, None], 0.0)
        k_dir = np.where(kn[:, None] > 0, kt / np.where(kn > 0, kn, 1.0)[:, None], 0.0)
        Ge = np.einsum("nij,nj->ni", G, e)                   # G e      (d_k)
        GTk = _read(G, kt)                                   # G^T k    (d_v)
        de = bt[:, None] * GTk + (dm[:, t] * bt * kn)[:, None] * e_dir
        dbeta[:, t] = np.einsum("ni,ni->n", kt, Ge) + dm[:, t] * kn * en
        dkk[:, t] = bt[:, None] * Ge + (dm[:, t] * bt * en)[:, None] * k_dir
        dkk[:, t] -= at[:, None] * np.einsum("nij,nj->ni", S_prev, de)
        dvv[:, t] = de
        da[:, t] = np.einsum("nij,nij->n", G, S_prev) - np.einsum("ni,nij,nj->n", kt, S_prev, de)
        G = at[:, None, None] * G - at[:, None, None] * kt[:, :, None] * de[:, None, :]
    return {
        "dq": dq.reshape(*lead, L, dk),
        "dk": dkk.reshape(*lead, L, dk),
        "dv": dvv.reshape(*lead, L, dv),
        "dbeta": dbeta.reshape(*lead, L),
        "da": da.reshape(*lead, L),
        "dS0": G.reshape(*lead, dk, dv),
    }


def scan_kalman_diag_backward(q, k, v, r, dO, a=None, qn=None, S0=None, p0=None, dm=None, dS_L=None, dp_L=None):
    """Gradients of the diagonal-Kalman scan (``oracle.scan.scan_kalman_diag``).

    Shapes: q, k [..., L, d_k]; v [..., L, d_v]; r, a, qn [..., L] (a, qn may be None: 1 and 0); S0
    [..., d_k, d_v]; p0 [..., d_k] (None = 1); upstream dO [..., L, d_v], dm [..., L], dS_L [..., d_k, d_v],
    dp_L [..., d_k] (each None = 0).  Returns dq, dk, dv, dr, da, dqn (per token), dS0 and dp0.
    """
    lead, n, L, dk, dv, q, k, v = _flatten_inputs(q, k, v)
    r = _per_token(r, n, L, 1.0)
    a = _per_token(a, n, L, 1.0)
    qn = _per_token(qn, n, L, 0.0)
    dO = _f64(dO).reshape(n, L, dv)
    dm = _per_token(dm, n, L, 0.0)
    S = np.zeros((n, dk, dv)) if S0 is None else _f64(S0).reshape(n, dk, dv).copy()
    p = np.ones((n, dk)) if p0 is None else _f64(p0).reshape(n, dk).copy()

    states = np.zeros((n, L + 1, dk, dv))
    pvec = np.zeros((n, L + 1, dk))
    states[:, 0], pvec[:, 0] = S, p
    res, gains, pms, ss = np.zeros((n, L, dv)), np.zeros((n, L, dk)), np.zeros((n, L, dk)), np.zeros((n, L))
    for t in range(L):
        kt, at = k[:, t], a[:, t]
        pm = (at * at)[:, None] * p + qn[:, t, None]
        st = np.einsum("ni,ni->n", pm, kt * kt) + r[:, t]
        g = pm * kt / st[:, None]
        p = pm * r[:, t, None] / (r[:, t, None] + pm * kt * kt)
        S_pred = at[:, None, None] * S
        e = v[:, t] - _read(S_pred, kt)
        S = S_pred + g[:, :, None] * e[:, None, :]
        states[:, t + 1], pvec[:, t + 1] = S, p
        res[:, t], gains[:, t], pms[:, t], ss[:, t] = e, g, pm, st

    G = np.zeros((n, dk, dv)) if dS_L is None else _f64(dS_L).reshape(n, dk, dv).copy()
    Pb = np.zeros((n, dk)) if dp_L is None else _f64(dp_L).reshape(n, dk).copy()
    dq, dkk, dvv = np.zeros((n, L, dk)), np.zeros((n, L, dk)), np.zeros((n, L, dv))
    dr, da, dqn = np.zeros((n, L)), np.zeros((n, L)), np.zeros((n, L))
    for t in range(L - 1, -1, -1):
        kt, qt, e, g, pm, st = k[:, t], q[:, t], res[:, t], gains[:, t], pms[:, t], ss[:, t]
        at, rt = a[:, t], r[:, t]
        S_t, S_prev, p_prev = states[:, t + 1], states[:, t], pvec[:, t]
        G = G + qt[:, :, None] * dO[:, t, None, :]
        dq[:, t] = np.einsum("nij,nj->ni", S_t, dO[:, t])
        gn = np.linalg.norm(g, axis=-1)
        en = np.linalg.norm(e, axis=-1)
        e_dir = np.where(en[:, None] > 0, e / np.where(en > 0, en, 1.0)[:, None], 0.0)
        g_dir = np.where(gn[:, None] > 0, g / np.where(gn > 0, gn, 1.0)[:, None], 0.0)
        # the write S_t = a S_{t-1} + g e^T and the surprise m_t = ||g|| ||e||
        de = _read(G, g) + (dm[:, t] * gn)[:, None] * e_dir
        dg = np.einsum("nij,nj->ni", G, e) + (dm[:, t] * en)[:, None] * g_dir
        dkt = -at[:, None] * np.einsum("nij,nj->ni", S_prev, de)
        dvv[:, t] = de
        da_t = np.einsum("nij,nij->n", G, S_prev) - np.einsum("ni,nij,nj->n", kt, S_prev, de)
        G = at[:, None, None] * G - at[:, None, None] * kt[:, :, None] * de[:, None, :]
        # g = p^- o k / s
        dpm = dg * kt / st[:, None]
        dkt += dg * pm / st[:, None]
        ds = -np.einsum("ni,ni->n", dg, g) / st
        # p = p^- r / (r + p^- k^2)
        den = rt[:, None] + pm * kt * kt
        dpm += Pb * rt[:, None] ** 2 / den ** 2
        dr_t = np.einsum("ni,ni->n", Pb, (pm * kt) ** 2 / den ** 2)
        dkt -= 2.0 * Pb * pm * pm * rt[:, None] * kt / den ** 2
        # s = sum p^- k^2 + r
        dpm += ds[:, None] * kt * kt
        dkt += 2.0 * ds[:, None] * pm * kt
        dr_t += ds
        # p^- = a^2 p + Qn
        Pb = (at * at)[:, None] * dpm
        da_t += 2.0 * at * np.einsum("ni,ni->n", dpm, p_prev)
        dqn[:, t] = dpm.sum(axis=-1)
        dkk[:, t], dr[:, t], da[:, t] = dkt, dr_t, da_t
    return {
        "dq": dq.reshape(*lead, L, dk),
        "dk": dkk.reshape(*lead, L, dk),
        "dv": dvv.reshape(*lead, L, dv),
        "dr": dr.reshape(*lead, L),
        "da": da.reshape(*lead, L),
        "dqn": dqn.reshape(*lead, L),
        "dS0": G.reshape(*lead, dk, dv),
        "dp0": Pb.reshape(*lead, dk),
    }


def _memory_step_backward(G, g, e, kt, qt, S_t, S_prev, at, dOt, dmt):
    """The memory part of one token's backward for a gain g (rows of heads): the read, the write
    S_t = a S_{t-1} + g e^T, the residual e = v - a S_{t-1}^T k and the surprise ||g|| ||e||.
    G enters as dLoss/dS_t without the read; returns (G_{t-1}, dq, dv, dk through the residual, da, dg)."""
    G = G + qt[:, :, None] * dOt[:, None, :]
    dq = np.einsum("nij,nj->ni", S_t, dOt)
    gn = np.linalg.norm(g, axis=-1)
    en = np.linalg.norm(e, axis=-1)
    e_dir = np.where(en[:, None] > 0, e / np.where(en > 0, en, 1.0)[:, None], 0.0)
    g_dir = np.where(gn[:, None] > 0, g / np.where(gn > 0, gn, 1.0)[:, None], 0.0)
    de = _read(G, g) + (dmt * gn)[:, None] * e_dir
    dg = np.einsum("nij,nj->ni", G, e) + (dmt * en)[:, None] * g_dir
    dk = -at[:, None] * np.einsum("nij,nj->ni", S_prev, de)
    da = np.einsum("nij,nij->n", G, S_prev) - np.einsum("ni,nij,nj->n", kt, S_prev, de)
    G = at[:, None, None] * G - at[:, None, None] * kt[:, :, None] * de[:, None, :]
    return G, dq, de, dk, da, dg


def scan_kalman_iso_backward(q, k, v, r, dO, a=None, qn=None, S0=None, c0=None, dm=None, dS_L=None, dc_L=None):
    """Gradients of the isotropic-Kalman scan (``oracle.scan.scan_kalman_iso``).  c0 [...] (None = 1) and
    upstream dc_L [...] (None = 0) are per head.  Returns dq, dk, dv, dr, da, dqn, dS0 and dc0."""
    lead, n, L, dk, dv, q, k, v = _flatten_inputs(q, k, v)
    r = _per_token(r, n, L, 1.0)
    a = _per_token(a, n, L, 1.0)
    qn = _per_token(qn, n, L, 0.0)
    dO = _f64(dO).reshape(n, L, dv)
    dm = _per_token(dm, n, L, 0.0)
    S = np.zeros((n, dk, dv)) if S0 is None else _f64(S0).reshape(n, dk, dv).copy()
    c = np.ones(n) if c0 is None else _f64(c0).reshape(n).copy()
    states, cs = np.zeros((n, L + 1, dk, dv)), np.zeros((n, L + 1))
    states[:, 0], cs[:, 0] = S, c
    res, gains = np.zeros((n, L, dv)), np.zeros((n, L, dk))
    for t in range(L):
        kt, at = k[:, t], a[:, t]
        cm = at * at * c + qn[:, t]
        kk = np.einsum("ni,ni->n", kt, kt)
        g = (cm / (cm * kk + r[:, t]))[:, None] * kt
        c = dk * cm * r[:, t] / (dk * r[:, t] + cm * kk)
        S_pred = at[:, None, None] * S
        e = v[:, t] - _read(S_pred, kt)
        S = S_pred + g[:, :, None] * e[:, None, :]
        states[:, t + 1], cs[:, t + 1], res[:, t], gains[:, t] = S, c, e, g
    G = np.zeros((n, dk, dv)) if dS_L is None else _f64(dS_L).reshape(n, dk, dv).copy()
    cb = np.zeros(n) if dc_L is None else _f64(dc_L).reshape(n).copy()
    out = {key: np.zeros(shape) for key, shape in
           (("dq", (n, L, dk)), ("dk", (n, L, dk)), ("dv", (n, L, dv)), ("dr", (n, L)), ("da", (n, L)),
            ("dqn", (n, L)))}
    for t in range(L - 1, -1, -1):
        kt, at, rt, c_prev = k[:, t], a[:, t], r[:, t], cs[:, t]
        G, dq, de, dkt, da_t, dg = _memory_step_backward(G, gains[:, t], res[:, t], kt, q[:, t], states[:, t + 1],
                                                         states[:, t], at, dO[:, t], dm[:, t])
        cm = at * at * c_prev + qn[:, t]
        kk = np.einsum("ni,ni->n", kt, kt)
        st = cm * kk + rt
        beta = cm / st
        # g = beta k, beta = c^- / s, s = c^- kk + r
        dbeta = np.einsum("ni,ni->n", kt, dg)
        dkt = dkt + beta[:, None] * dg
        dcm = dbeta / st
        ds = -dbeta * cm / st ** 2
        dcm = dcm + ds * kk
        dkk = ds * cm
        dr_t = ds
        # c = d c^- r / (d r + c^- kk)
        den = dk * rt + cm * kk
        dcm = dcm + cb * (dk * rt) ** 2 / den ** 2
        dr_t = dr_t + cb * dk * cm * cm * kk / den ** 2
        dkk = dkk - cb * dk * cm * cm * rt / den ** 2
        dkt = dkt + 2.0 * dkk[:, None] * kt
        # c^- = a^2 c + Qn
        cb = at * at * dcm
        da_t = da_t + 2.0 * at * c_prev * dcm
        out["dq"][:, t], out["dk"][:, t], out["dv"][:, t] = dq, dkt, de
        out["dr"][:, t], out["da"][:, t], out["dqn"][:, t] = dr_t, da_t, dcm
    res_out = {key: val.reshape(*lead, *val.shape[1:]) for key, val in out.items()}
    res_out["dS0"] = G.reshape(*lead, dk, dv)
    res_out["dc0"] = cb.reshape(lead)
    return res_out


def scan_kalman_full_backward(q, k, v, r, dO, a=None, qn=None, S0=None, P0=None, dm=None, dS_L=None, dP_L=None):
    """Gradients of the full-covariance Kalman scan (``oracle.scan.scan_kalman_full``).  P0 [..., d_k, d_k]
    (None = I), upstream dP_L [..., d_k, d_k] (None = 0).  Returns dq, dk, dv, dr, da, dqn, dS0 and dP0 (the
    gradient with respect to every entry of P0, as the forward uses it)."""
    lead, n, L, dk, dv, q, k, v = _flatten_inputs(q, k, v)
    r = _per_token(r, n, L, 1.0)
    a = _per_token(a, n, L, 1.0)
    qn = _per_token(qn, n, L, 0.0)
    dO = _f64(dO).reshape(n, L, dv)
    dm = _per_token(dm, n, L, 0.0)
    eye = np.eye(dk)
    S = np.zeros((n, dk, dv)) if S0 is None else _f64(S0).reshape(n, dk, dv).copy()
    P = np.broadcast_to(eye, (n, dk, dk)).copy() if P0 is None else _f64(P0).reshape(n, dk, dk).copy()
    states, Ps = np.zeros((n, L + 1, dk, dv)), np.zeros((n, L + 1, dk, dk))
    states[:, 0], Ps[:, 0] = S, P
    res, gains = np.zeros((n, L, dv)), np.zeros((n, L, dk))
    for t in range(L):
        kt, at = k[:, t], a[:, t]
        Pm = (at * at)[:, None, None] * P + qn[:, t, None, None] * eye
        u = np.einsum("nij,nj->ni", Pm, kt)
        st = np.einsum("ni,ni->n", kt, u) + r[:, t]
        g = u / st[:, None]
        P = Pm - u[:, :, None] * u[:, None, :] / st[:, None, None]
        S_pred = at[:, None, None] * S
        e = v[:, t] - _read(S_pred, kt)
        S = S_pred + g[:, :, None] * e[:, None, :]
        states[:, t + 1], Ps[:, t + 1], res[:, t], gains[:, t] = S, P, e, g
    G = np.zeros((n, dk, dv)) if dS_L is None else _f64(dS_L).reshape(n, dk, dv).copy()
    Pb = np.zeros((n, dk, dk)) if dP_L is None else _f64(dP_L).reshape(n, dk, dk).copy()
    out = {key: np.zeros(shape) for key, shape in
           (("dq", (n, L, dk)), ("dk", (n, L, dk)), ("dv", (n, L, dv)), ("dr", (n, L)), ("da", (n, L)),
            ("dqn", (n, L)))}
    for t in range(L - 1, -1, -1):
        kt, at, rt, P_prev = k[:, t], a[:, t], r[:, t], Ps[:, t]
        G, dq, de, dkt, da_t, dg = _memory_step_backward(G, gains[:, t], res[:, t], kt, q[:, t], states[:, t + 1],
                                                         states[:, t], at, dO[:, t], dm[:, t])
        Pm = (at * at)[:, None, None] * P_prev + qn[:, t, None, None] * eye
        u = np.einsum("nij,nj->ni", Pm, kt)
        st = np.einsum("ni,ni->n", kt, u) + rt
        g = u / st[:, None]
        # g = u / s
        du = dg / st[:, None]
        ds = -np.einsum("ni,ni->n", dg, g) / st
        # P = P^- - u u^T / s
        dPm = Pb.copy()
        du = du - np.einsum("nij,nj->ni", Pb + np.swapaxes(Pb, 1, 2), u) / st[:, None]
        ds = ds + np.einsum("ni,nij,nj->n", u, Pb, u) / st ** 2
        # s = k^T u + r
        dkt = dkt + ds[:, None] * u
        du = du + ds[:, None] * kt
        dr_t = ds
        # u = P^- k
        dPm = dPm + du[:, :, None] * kt[:, None, :]
        dkt = dkt + np.einsum("nji,nj->ni", Pm, du)
        # P^- = a^2 P + Qn I
        Pb = (at * at)[:, None, None] * dPm
        da_t = da_t + 2.0 * at * np.einsum("nij,nij->n", dPm, P_prev)
        out["dq"][:, t], out["dk"][:, t], out["dv"][:, t] = dq, dkt, de
        out["dr"][:, t], out["da"][:, t], out["dqn"][:, t] = dr_t, da_t, np.trace(dPm, axis1=1, axis2=2)
    res_out = {key: val.reshape(*lead, *val.shape[1:]) for key, val in out.items()}
    res_out["dS0"] = G.reshape(*lead, dk, dv)
    res_out["dP0"] = Pb.reshape(*lead, dk, dk)
    return res_out
