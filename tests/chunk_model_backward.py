"""Float64 NumPy model of the chunked backward of the four scans.

Test infrastructure, like ``tests/chunk_model.py``: it checks the reverse-mode algebra of the chunk form
against the token-by-token backward oracle (``oracle.backward``) before any kernel exists, so that a
tensor-core backward can follow it block by block.  It shares no code with the oracle or the product.

Forward of one chunk of n tokens from the state S0 (G = diag(beta) K; lower = with the diagonal):

    ell_i = sum_{m<=i} log a_m,  A_i = exp(ell_i),  Gam_ij = exp(ell_i - ell_j) (i >= j),
    r_j = A_C / A_j,  A_C = A_{n-1}
    N = strict_lower((K G^T) o Gam),  T = (I + N)^-1,  M = lower((Q G^T) o Gam),  AT = M T
    R = V - diag(A) K S0,  E = T R,  O = diag(A) Q S0 + AT R,
    S_C = A_C S0 + G^T diag(r) E,    m_j = beta_j ||k_j|| ||e_j||

Backward of the chunk for upstream dO, dm and dS_C, every product a dense matrix product:

    dS0 = A_C dS_C + Q^T diag(A) dO - K^T diag(A) dR,   dE = diag(r) G dS_C + (surprise term)
    dR  = AT^T dO + T^T dE,   dT = dE R^T + M^T dAT,   dAT = dO R^T,   dM = dAT T^T
    dN  = strict_lower(-T^T dT T^T)
    d(K G^T) = dN o Gam,  d(Q G^T) = lower(dM) o Gam,  dGam = dN o (K G^T) + lower(dM) o (Q G^T)
    dV = dR,  dQ = diag(A) dO S0^T + d(Q G^T) G,  dK = -diag(A) dR S0^T + d(K G^T) G + diag(beta) dG,
    dG = d(K G^T)^T K + d(Q G^T)^T Q + diag(r) E dS_C^T,  dbeta_j = k_j . dG_j
and the gate terms collect in log space: dell_i = A_i dA_i + sum_j Gam_ij dGam_ij - sum_i' Gam_i'i dGam_i'i
- r_i dr_i (plus A_C dA_C + sum_j r_j dr_j at i = n - 1), d log a_m = sum_{i >= m} dell_i, da = d log a / a.
The chunk's dS0 is the previous chunk's dS_C.  For the diagonal variant G holds the Kalman gains; dG then
runs back through the per-token variance recursion that made them (sequential within a chunk, as in the
forward), with the variance adjoint carried from chunk to chunk; the isotropic variant runs dbeta back through
its scalar recursion.  For full Kalman dG runs back through the chunk's covariance side: the rank-n update
P_C = A_C^2 P0 + gamma_C I - G^T diag(w) G, the gains G = Z / D, Z = (L^-1 o Gam) Bt, the inverse
(dL = -L^-T dLinv L^-T), the LDL of the innovation Gram (dG = L^-T M L^-1 with
M = strict_lower(L^T dL D^-1) + diag(dD)), the Gram and Bt = diag(A^2) K P0 + diag(gamma) K; the covariance
adjoint goes to the previous chunk.
"""

import numpy as np


def _gates(a_chunk):
    ell = np.cumsum(np.log(a_chunk))
    gam = np.tril(np.exp(ell[:, None] - ell[None, :]))
    return ell, np.exp(ell), gam


def _wy_chunk_backward(Qc, Kc, Vc, G, ac, S0c, dOc, dmc, dS):
    """Backward of one chunk of the generalised WY form for gains G (rows g_j) and surprise
    m_j = ||g_j|| ||e_j||.  Returns dQ, dK (through the products only), dV, dG, d log a, dS0."""
    n, dk = Kc.shape
    ell, A, gam = _gates(ac)
    AC = A[-1]
    rr = AC / A
    KG, QG = Kc @ G.T, Qc @ G.T
    N = np.tril(KG * gam, -1)
    T = np.linalg.inv(np.eye(n) + N)
    Mm = np.tril(QG * gam)
    AT = Mm @ T
    KS, QS = Kc @ S0c, Qc @ S0c
    R = Vc - A[:, None] * KS
    E = T @ R
    W = (G * rr[:, None]).T                                   # d_k x n
    # S_C = A_C S0 + W E
    dS0 = AC * dS
    dAC = np.sum(dS * S0c)
    dW = dS @ E.T
    dE = W.T @ dS
    # surprise m_j = ||g_j|| ||e_j||
    gn, en = np.linalg.norm(G, axis=1), np.linalg.norm(E, axis=1)
    dG = np.zeros_like(G)
    nz = en > 0
    dE[nz] += (dmc * gn)[nz, None] * E[nz] / en[nz, None]
    nzg = gn > 0
    dG[nzg] += (dmc * en)[nzg, None] * G[nzg] / gn[nzg, None]
    # O = diag(A) Q S0 + AT R
    dA = np.sum(dOc * QS, axis=1)
    dQS = A[:, None] * dOc
    dQc = dQS @ S0c.T
    dS0 += Qc.T @ dQS
    dAT = dOc @ R.T
    dR = AT.T @ dOc
    # E = T R
    dR += T.T @ dE
    dT = dE @ R.T
    # AT = M T
    dM = np.tril(dAT @ T.T)
    dT += Mm.T @ dAT
    # T = (I + N)^-1
    dN = np.tril(-T.T @ dT @ T.T, -1)
    dKG = dN * gam
    dQG = dM * gam
    dGam = dN * KG + dM * QG
    # R = V - diag(A) K S0
    dVc = dR
    dA -= np.sum(dR * KS, axis=1)
    dKS = -A[:, None] * dR
    dKc = dKS @ S0c.T
    dS0 += Kc.T @ dKS
    # K G^T, Q G^T, W = G^T diag(r)
    dKc += dKG @ G
    dQc += dQG @ G
    dG += dKG.T @ Kc + dQG.T @ Qc + rr[:, None] * dW.T
    drr = np.sum(G * dW.T, axis=1)
    # gates in log space
    dell = A * dA + np.sum(gam * dGam, axis=1) - np.sum(gam * dGam, axis=0) - rr * drr
    dell[-1] += AC * dAC + np.sum(rr * drr)
    dloga = np.cumsum(dell[::-1])[::-1]
    return dQc, dKc, dVc, dG, dloga, dS0


def _wy_chunk_forward(Kc, Vc, G, ac, S):
    n = Kc.shape[0]
    _, A, gam = _gates(ac)
    N = np.tril((Kc @ G.T) * gam, -1)
    T = np.linalg.inv(np.eye(n) + N)
    E = T @ (Vc - A[:, None] * (Kc @ S))
    return A[-1] * S + (G * (A[-1] / A)[:, None]).T @ E


def chunk_delta_backward(q, k, v, beta, a, C, dO, S0=None, dm=None, dS_L=None):
    """One head: q, k [L, dk], v [L, dv], beta, a [L] (a > 0), dO [L, dv], dm [L] or None, dS_L [dk, dv] or
    None.  Returns dq, dk, dv, dbeta, da, dS0 from the chunk form with chunks of C tokens."""
    L, dk = k.shape
    dv = v.shape[1]
    dm = np.zeros(L) if dm is None else np.asarray(dm, float)
    S = np.zeros((dk, dv)) if S0 is None else np.array(S0, float)
    chunks = [(c0, min(c0 + C, L)) for c0 in range(0, L, C)]
    starts = []
    for c0, c1 in chunks:
        starts.append(S.copy())
        S = _wy_chunk_forward(k[c0:c1], v[c0:c1], beta[c0:c1, None] * k[c0:c1], a[c0:c1], S)
    dS = np.zeros((dk, dv)) if dS_L is None else np.array(dS_L, float)
    dq, dkk, dvv = np.zeros((L, dk)), np.zeros((L, dk)), np.zeros((L, dv))
    dbeta, da = np.zeros(L), np.zeros(L)
    for (c0, c1), S0c in reversed(list(zip(chunks, starts))):
        Kc, bc = k[c0:c1], beta[c0:c1]
        dQc, dKc, dVc, dG, dloga, dS = _wy_chunk_backward(q[c0:c1], Kc, v[c0:c1], bc[:, None] * Kc, a[c0:c1], S0c,
                                                          dO[c0:c1], dm[c0:c1], dS)
        # G = diag(beta) K
        dq[c0:c1], dvv[c0:c1] = dQc, dVc
        dkk[c0:c1] = dKc + bc[:, None] * dG
        dbeta[c0:c1] = np.sum(Kc * dG, axis=1)
        da[c0:c1] = dloga / a[c0:c1]
    return {"dq": dq, "dk": dkk, "dv": dvv, "dbeta": dbeta, "da": da, "dS0": dS}


def chunk_diag_backward(q, k, v, r, a, qn, C, dO, S0=None, p0=None, dm=None, dS_L=None, dp_L=None):
    """Diagonal Kalman, one head: the chunk backward above for the gains, then the per-token adjoint of
    the variance recursion that made them (sequential within the chunk, like the forward's variances; the
    variance adjoint is carried across chunks).  Returns dq, dk, dv, dr, da, dqn, dS0, dp0."""
    L, dk = k.shape
    dv = v.shape[1]
    dm = np.zeros(L) if dm is None else np.asarray(dm, float)
    S = np.zeros((dk, dv)) if S0 is None else np.array(S0, float)
    p = np.ones(dk) if p0 is None else np.array(p0, float)
    chunks = [(c0, min(c0 + C, L)) for c0 in range(0, L, C)]
    starts, pstarts, gains = [], [], []
    for c0, c1 in chunks:
        starts.append(S.copy())
        pstarts.append(p.copy())
        G = np.zeros((c1 - c0, dk))
        for i, t in enumerate(range(c0, c1)):
            pm = a[t] ** 2 * p + qn[t]
            G[i] = pm * k[t] / (pm @ (k[t] ** 2) + r[t])
            p = pm * r[t] / (r[t] + pm * k[t] ** 2)
        gains.append(G)
        S = _wy_chunk_forward(k[c0:c1], v[c0:c1], G, a[c0:c1], S)
    dS = np.zeros((dk, dv)) if dS_L is None else np.array(dS_L, float)
    Pb = np.zeros(dk) if dp_L is None else np.array(dp_L, float)
    out = {key: np.zeros(shape) for key, shape in
           (("dq", (L, dk)), ("dk", (L, dk)), ("dv", (L, dv)), ("dr", L), ("da", L), ("dqn", L))}
    for ci in range(len(chunks) - 1, -1, -1):
        c0, c1 = chunks[ci]
        G = gains[ci]
        dQc, dKc, dVc, dG, dloga, dS = _wy_chunk_backward(q[c0:c1], k[c0:c1], v[c0:c1], G, a[c0:c1], starts[ci],
                                                          dO[c0:c1], dm[c0:c1], dS)
        out["dq"][c0:c1], out["dv"][c0:c1] = dQc, dVc
        da_c = dloga / a[c0:c1]
        # the variance recursion of this chunk, replayed to recover p before each token, then reversed
        pp = [pstarts[ci]]
        for t in range(c0, c1 - 1):
            pm = a[t] ** 2 * pp[-1] + qn[t]
            pp.append(pm * r[t] / (r[t] + pm * k[t] ** 2))
        for i in range(c1 - c0 - 1, -1, -1):
            t = c0 + i
            kt, pprev = k[t], pp[i]
            pm = a[t] ** 2 * pprev + qn[t]
            st = pm @ (kt ** 2) + r[t]
            g = pm * kt / st
            dg = dG[i]
            dpm = dg * kt / st
            dKc[i] += dg * pm / st
            ds = -(dg @ g) / st
            den = r[t] + pm * kt ** 2
            dpm += Pb * r[t] ** 2 / den ** 2 + ds * kt ** 2
            out["dr"][t] += np.sum(Pb * (pm * kt) ** 2 / den ** 2) + ds
            dKc[i] += -2.0 * Pb * pm * pm * r[t] * kt / den ** 2 + 2.0 * ds * pm * kt
            Pb = a[t] ** 2 * dpm
            da_c[i] += 2.0 * a[t] * (dpm @ pprev)
            out["dqn"][t] = dpm.sum()
        out["dk"][c0:c1] = dKc
        out["da"][c0:c1] = da_c
    out["dS0"], out["dp0"] = dS, Pb
    return out


def chunk_iso_backward(q, k, v, r, a, qn, C, dO, S0=None, c0=1.0, dm=None, dS_L=None, dc_L=0.0):
    """Isotropic Kalman, one head: the delta chunk backward for beta_t = c^-_t / (c^-_t ||k_t||^2 + r_t), then
    the per-token adjoint of the uncertainty scalar's recursion.  Returns dq, dk, dv, dr, da, dqn, dS0, dc0."""
    L, dk = k.shape
    kk = np.sum(k * k, axis=1)
    c = float(c0)
    cprev, beta = np.zeros(L), np.zeros(L)
    for t in range(L):
        cprev[t] = c
        cm = a[t] ** 2 * c + qn[t]
        beta[t] = cm / (cm * kk[t] + r[t])
        c = dk * cm * r[t] / (dk * r[t] + cm * kk[t])
    g = chunk_delta_backward(q, k, v, beta, a, C, dO, S0=S0, dm=dm, dS_L=dS_L)
    out = {"dq": g["dq"], "dk": g["dk"].copy(), "dv": g["dv"], "da": g["da"].copy(), "dS0": g["dS0"],
           "dr": np.zeros(L), "dqn": np.zeros(L)}
    cb = float(dc_L)
    for t in range(L - 1, -1, -1):
        cm = a[t] ** 2 * cprev[t] + qn[t]
        st = cm * kk[t] + r[t]
        db = g["dbeta"][t]
        dcm = db / st - db * cm / st ** 2 * kk[t]
        dkk = -db * cm / st ** 2 * cm
        dr = -db * cm / st ** 2
        den = dk * r[t] + cm * kk[t]
        dcm += cb * (dk * r[t]) ** 2 / den ** 2
        dr += cb * dk * cm * cm * kk[t] / den ** 2
        dkk -= cb * dk * cm * cm * r[t] / den ** 2
        out["dk"][t] += 2.0 * dkk * k[t]
        out["dr"][t] = dr
        out["dqn"][t] = dcm
        out["da"][t] += 2.0 * a[t] * cprev[t] * dcm
        cb = a[t] ** 2 * dcm
    out["dc0"] = cb
    return out


def _ldl(G):
    n = G.shape[0]
    L = np.eye(n)
    D = np.zeros(n)
    A = G.copy()
    for j in range(n):
        D[j] = A[j, j]
        L[j + 1:, j] = A[j + 1:, j] / D[j]
        A[j + 1:, j + 1:] -= np.outer(L[j + 1:, j], L[j + 1:, j]) * D[j]
    return L, D


def ldl_backward(L, D, dL, dD):
    """Adjoint of G = L D L^T (L unit lower) as a function of the lower triangle of the symmetric G.
    With X = L^-1 dG L^-T (symmetric), dD = diag(X) and dL = L strict_lower(X) D^-1, so for upstream dL
    (strict lower) and dD the matrix M = strict_lower(L^T dL D^-1) + diag(dD) gives dG = L^-T M L^-1 over
    symmetric perturbations; an entry below the diagonal stands for both of its mirror images."""
    Li = np.linalg.inv(L)
    M = np.tril(L.T @ np.tril(dL, -1) / D[None, :], -1) + np.diag(dD)
    Gb = Li.T @ M @ Li
    return np.tril(Gb + Gb.T, -1) + np.diag(np.diag(Gb))


def chunk_full_backward(q, k, v, r, a, qn, C, dO, S0=None, P0=None, dm=None, dS_L=None, dP_L=None):
    """Full-covariance Kalman, one head: the WY chunk backward for the gains, then the adjoint of the
    chunk's covariance side (Gram, LDL, L^-1, Z, the rank-n covariance update), with the covariance adjoint
    carried from chunk to chunk.  P0 symmetric; returns dq, dk, dv, dr, da, dqn, dS0 and dP0 (symmetric)."""
    L, dk = k.shape
    dv = v.shape[1]
    dm = np.zeros(L) if dm is None else np.asarray(dm, float)
    S = np.zeros((dk, dv)) if S0 is None else np.array(S0, float)
    P = np.eye(dk) if P0 is None else np.array(P0, float)
    eye = np.eye(dk)
    chunks = [(c0, min(c0 + C, L)) for c0 in range(0, L, C)]

    def cov_forward(Kc, ac, qnc, rc, P):
        n = Kc.shape[0]
        ell, A, gam = _gates(ac)
        gamma = np.zeros(n)
        gp = 0.0
        for i in range(n):
            gp = ac[i] ** 2 * gp + qnc[i]
            gamma[i] = gp
        KP = Kc @ P
        Bt = (A ** 2)[:, None] * KP + gamma[:, None] * Kc
        Graw = Kc @ Bt.T
        low = np.tril(Graw * gam) + np.diag(rc)
        Gs = low + np.tril(low, -1).T
        Lf, D = _ldl(Gs)
        Li = np.linalg.inv(Lf)
        Y = Li * gam
        Z = Y @ Bt
        Gm = Z / D[:, None]
        rr = A[-1] / A
        w = rr ** 2 * D
        PC = A[-1] ** 2 * P + gamma[-1] * eye - (Gm.T * w) @ Gm
        return dict(ell=ell, A=A, gam=gam, gamma=gamma, KP=KP, Bt=Bt, Graw=Graw, Lf=Lf, D=D, Li=Li, Y=Y, Z=Z,
                    Gm=Gm, rr=rr, w=w, PC=0.5 * (PC + PC.T))

    starts, Pstarts, caches = [], [], []
    for c0, c1 in chunks:
        starts.append(S.copy())
        Pstarts.append(P.copy())
        cf = cov_forward(k[c0:c1], a[c0:c1], qn[c0:c1], r[c0:c1], P)
        caches.append(cf)
        P = cf["PC"]
        S = _wy_chunk_forward(k[c0:c1], v[c0:c1], cf["Gm"], a[c0:c1], S)

    dS = np.zeros((dk, dv)) if dS_L is None else np.array(dS_L, float)
    dP = np.zeros((dk, dk)) if dP_L is None else np.array(dP_L, float)
    out = {key: np.zeros(shape) for key, shape in
           (("dq", (L, dk)), ("dk", (L, dk)), ("dv", (L, dv)), ("dr", L), ("da", L), ("dqn", L))}
    for ci in range(len(chunks) - 1, -1, -1):
        c0, c1 = chunks[ci]
        cf, P0c = caches[ci], Pstarts[ci]
        Kc, ac = k[c0:c1], a[c0:c1]
        n = c1 - c0
        A, gam, rr, D, Gm = cf["A"], cf["gam"], cf["rr"], cf["D"], cf["Gm"]
        AC = A[-1]
        dQc, dKc, dVc, dGm, dloga, dS = _wy_chunk_backward(q[c0:c1], Kc, v[c0:c1], Gm, ac, starts[ci], dO[c0:c1],
                                                           dm[c0:c1], dS)
        # P_C = sym(A_C^2 P0 + gamma_C I - Gm^T diag(w) Gm)
        dPC = 0.5 * (dP + dP.T)
        dP0 = AC ** 2 * dPC
        dA = np.zeros(n)
        dAC = 2.0 * AC * np.sum(dPC * P0c)
        dgamma = np.zeros(n)
        dgamma[-1] += np.trace(dPC)
        dGm -= (cf["w"][:, None] * Gm) @ (dPC + dPC.T)
        dw = -np.einsum("ji,ik,jk->j", Gm, dPC, Gm)
        dD = dw * rr ** 2
        drr = dw * 2.0 * rr * D
        # Gm = Z / D
        dZ = dGm / D[:, None]
        dD -= np.sum(dGm * Gm, axis=1) / D
        # Z = Y Bt, Y = L^-1 o Gam
        dY = dZ @ cf["Bt"].T
        dBt = cf["Y"].T @ dZ
        dLi = np.tril(dY * gam)
        dgam = np.tril(dY * cf["Li"])
        # L^-1 from L
        dLf = np.tril(-cf["Li"].T @ dLi @ cf["Li"].T, -1)
        # LDL, then the Gram's lower part: tril(Graw o Gam) + diag(r)
        dlow = ldl_backward(cf["Lf"], D, dLf, dD)
        out["dr"][c0:c1] = np.diag(dlow)
        dGraw = dlow * gam
        dgam += dlow * cf["Graw"]
        # Graw = K Bt^T
        dKc += dGraw @ cf["Bt"]
        dBt += dGraw.T @ Kc
        # Bt = diag(A^2) K P0 + diag(gamma) K
        dKP = (A ** 2)[:, None] * dBt
        dKc += dKP @ P0c.T + cf["gamma"][:, None] * dBt
        dP0 += Kc.T @ dKP
        dA += 2.0 * A * np.sum(dBt * cf["KP"], axis=1)
        dgamma += np.sum(dBt * Kc, axis=1)
        # gamma_j = a_j^2 gamma_{j-1} + Qn_j
        da_c = np.zeros(n)
        for j in range(n - 1, -1, -1):
            out["dqn"][c0 + j] = dgamma[j]
            gprev = cf["gamma"][j - 1] if j > 0 else 0.0
            da_c[j] += 2.0 * ac[j] * gprev * dgamma[j]
            if j > 0:
                dgamma[j - 1] += ac[j] ** 2 * dgamma[j]
        # gates of the covariance side, in log space
        dell = A * dA + np.sum(gam * dgam, axis=1) - np.sum(gam * dgam, axis=0) - rr * drr
        dell[-1] += AC * dAC + np.sum(rr * drr)
        dloga = dloga + np.cumsum(dell[::-1])[::-1]
        out["dq"][c0:c1], out["dk"][c0:c1], out["dv"][c0:c1] = dQc, dKc, dVc
        out["da"][c0:c1] = dloga / ac + da_c
        dP = dP0
    out["dS0"], out["dP0"] = dS, 0.5 * (dP + dP.T)
    return out


def full_cov_backward_tokens(k, r, a, qn, P0, dg, dP_L=None, block=64):
    """Full-covariance Kalman, one head: the covariance side of the backward token by token, as the CUDA
    kernels take it, for the gains' upstream gradient dg [L, d_k] from the memory backward.

    The forward P^- = a^2 P + Qn I, u = P^- k, s = k^T u + r, g = u / s, P <- P^- - u u^T / s keeps P at every
    block start; the backward recomputes each block's P, u, s from its checkpoint and walks it in reverse.
    Instead of the covariance adjoint Pb it carries M = Pb + Pb^T, which is enough while P is symmetric:
    (Pb + Pb^T) u = M u, u^T Pb u = u^T M u / 2, <Pb, P> = <M, P> / 2, tr Pb = tr M / 2, and
    Pb <- a^2 (Pb + du k^T) becomes the symmetric M <- a^2 (M + du k^T + k du^T).  Returns the covariance
    side's key and gate terms (dk, da: to be added to the memory backward's), dr, dqn and dP0 = M_0 / 2, the
    gradient with respect to a symmetric P0."""
    L, d = k.shape
    eye = np.eye(d)
    P = np.array(P0, float)
    ckpt = []
    for t in range(L):
        if t % block == 0:
            ckpt.append(P.copy())
        Pm = a[t] ** 2 * P + qn[t] * eye
        u = Pm @ k[t]
        P = Pm - np.outer(u, u) / (k[t] @ u + r[t])
    M = np.zeros((d, d)) if dP_L is None else np.array(dP_L, float) + np.array(dP_L, float).T
    trM = np.trace(M)
    out = {key: np.zeros(shape) for key, shape in (("dk", (L, d)), ("da", L), ("dr", L), ("dqn", L))}
    for b in range(len(ckpt) - 1, -1, -1):
        t0, t1 = b * block, min(L, (b + 1) * block)
        P = ckpt[b].copy()
        Pp, U, S = [], [], []
        for t in range(t0, t1):
            Pp.append(P)
            Pm = a[t] ** 2 * P + qn[t] * eye
            u = Pm @ k[t]
            s = k[t] @ u + r[t]
            U.append(u)
            S.append(s)
            P = Pm - np.outer(u, u) / s
        for t in range(t1 - 1, t0 - 1, -1):
            Pprev, u, s, kt = Pp[t - t0], U[t - t0], S[t - t0], k[t]
            Mu, Pk = M @ u, Pprev @ kt
            ds = (-(dg[t] @ u) + 0.5 * (u @ Mu)) / s ** 2
            du = (dg[t] - Mu) / s + ds * kt
            out["dk"][t] = ds * u + a[t] ** 2 * (Pprev @ du) + qn[t] * du
            out["da"][t] = 2.0 * a[t] * (0.5 * np.sum(M * Pprev) + du @ Pk)
            out["dqn"][t] = 0.5 * trM + du @ kt
            out["dr"][t] = ds
            M = a[t] ** 2 * (M + np.outer(du, kt) + np.outer(kt, du))
            trM = a[t] ** 2 * (trM + 2.0 * (du @ kt))
    out["dP0"] = 0.5 * M
    return out
