"""Float64 NumPy model of the chunked backward of the gated delta rule.

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
The chunk's dS0 is the previous chunk's dS_C.
"""

import numpy as np


def _gates(a_chunk):
    ell = np.cumsum(np.log(a_chunk))
    gam = np.tril(np.exp(ell[:, None] - ell[None, :]))
    return ell, np.exp(ell), gam


def chunk_delta_backward(q, k, v, beta, a, C, dO, S0=None, dm=None, dS_L=None):
    """One head: q, k [L, dk], v [L, dv], beta, a [L] (a > 0), dO [L, dv], dm [L] or None, dS_L [dk, dv] or
    None.  Returns dq, dk, dv, dbeta, da, dS0 from the chunk form with chunks of C tokens."""
    L, dk = k.shape
    dv = v.shape[1]
    dm = np.zeros(L) if dm is None else np.asarray(dm, float)
    S = np.zeros((dk, dv)) if S0 is None else np.array(S0, float)
    chunks = [(c0, min(c0 + C, L)) for c0 in range(0, L, C)]
    # forward in chunk form, keeping each chunk's start state
    starts = []
    for c0, c1 in chunks:
        starts.append(S.copy())
        Kc, Vc, bc = k[c0:c1], v[c0:c1], beta[c0:c1]
        n = c1 - c0
        _, A, gam = _gates(a[c0:c1])
        G = bc[:, None] * Kc
        N = np.tril((Kc @ G.T) * gam, -1)
        T = np.linalg.inv(np.eye(n) + N)
        E = T @ (Vc - A[:, None] * (Kc @ S))
        S = A[-1] * S + (G * (A[-1] / A)[:, None]).T @ E
    dS = np.zeros((dk, dv)) if dS_L is None else np.array(dS_L, float)
    dq, dkk, dvv = np.zeros((L, dk)), np.zeros((L, dk)), np.zeros((L, dv))
    dbeta, da = np.zeros(L), np.zeros(L)
    for (c0, c1), S0c in reversed(list(zip(chunks, starts))):
        Qc, Kc, Vc, bc, ac = q[c0:c1], k[c0:c1], v[c0:c1], beta[c0:c1], a[c0:c1]
        dOc, dmc = dO[c0:c1], dm[c0:c1]
        n = c1 - c0
        ell, A, gam = _gates(ac)
        AC = A[-1]
        rr = AC / A
        G = bc[:, None] * Kc
        KG, QG = Kc @ G.T, Qc @ G.T
        N = np.tril(KG * gam, -1)
        T = np.linalg.inv(np.eye(n) + N)
        Mm = np.tril(QG * gam)
        AT = Mm @ T
        KS, QS = Kc @ S0c, Qc @ S0c
        R = Vc - A[:, None] * KS
        E = T @ R
        W = (G * rr[:, None]).T                               # d_k x n
        # S_C = A_C S0 + W E
        dS0 = AC * dS
        dAC = np.sum(dS * S0c)
        dW = dS @ E.T
        dE = W.T @ dS
        # surprise m_j = beta_j ||k_j|| ||e_j||
        kn, en = np.linalg.norm(Kc, axis=1), np.linalg.norm(E, axis=1)
        dKc = np.zeros((n, dk))
        dbc = dmc * kn * en
        nz = en > 0
        dE[nz] += (dmc * bc * kn)[nz, None] * E[nz] / en[nz, None]
        nzk = kn > 0
        dKc[nzk] += (dmc * bc * en)[nzk, None] * Kc[nzk] / kn[nzk, None]
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
        dKc += dKS @ S0c.T
        dS0 += Kc.T @ dKS
        # K G^T, Q G^T, W = G^T diag(r), G = diag(beta) K
        dKc += dKG @ G
        dQc += dQG @ G
        dG = dKG.T @ Kc + dQG.T @ Qc + rr[:, None] * dW.T
        drr = np.sum(G * dW.T, axis=1)
        dbc += np.sum(Kc * dG, axis=1)
        dKc += bc[:, None] * dG
        # gates in log space
        dell = A * dA + np.sum(gam * dGam, axis=1) - np.sum(gam * dGam, axis=0) - rr * drr
        dell[-1] += AC * dAC + np.sum(rr * drr)
        dloga = np.cumsum(dell[::-1])[::-1]
        dq[c0:c1], dkk[c0:c1], dvv[c0:c1] = dQc, dKc, dVc
        dbeta[c0:c1] = dbc
        da[c0:c1] = dloga / ac
        dS = dS0
    return {"dq": dq, "dk": dkk, "dv": dvv, "dbeta": dbeta, "da": da, "dS0": dS}
