"""Float64 NumPy model of the chunked (blocked) forms the CUDA kernels compute.

Test infrastructure: it exists to check the chunk algebra against the
token-by-token oracle before and beside the kernels.  It is neither the oracle
nor the product, and shares no code with either.

Within a chunk of C tokens starting from S0 (and P0 / p0):
  ell_i = sum_{m<=i} log a_m, A_i = exp(ell_i), Gam_ij = A_i / A_j (i >= j)
  gains g_i (rows of Gm, C x d_k) come from the variant:
      delta   g_i = beta_i k_i
      diag    per-coordinate p recursion (no dependence on v or S)
      full    innovation Gram of the chunk and its LDL (Woodbury form), below
  then, for every variant (generalised WY / UT form):
      (I + strict_lower((K Gm^T) o Gam)) E = V - diag(A) K S0
      O   = diag(A) Q S0 + ((Q Gm^T) o Gam o lower_incl) E
      S_C = A_C S0 + Gm^T diag(A_C / A_j) E
      m_i = ||g_i|| ||e_i||
Full Kalman gains (joint Gaussian of the chunk):
  gamma_j = a_j^2 gamma_{j-1} + Qn_j, Pi_j = A_j^2 P0 + gamma_j I, Bt_j = Pi_j k_j
  G_ij = Gam_ij k_i^T Bt_j (i >= j, symmetric), G_ii += r_i;  G = L D L^T
  Z = (L^-1 o Gam) Bt  -> g_t = Z_t / D_t,  s_t = D_t
  P_C = Pi_C - sum_j (A_C/A_j)^2 s_j g_j g_j^T
"""

import numpy as np

LOG_A_FLOOR = -60.0  # a gate of 0 (a full reset) enters the log-space cumsum as exp(-60)


def _gates(a_chunk):
    la = np.log(np.maximum(a_chunk, np.exp(LOG_A_FLOOR)))
    ell = np.cumsum(la)
    gam = np.exp(ell[:, None] - ell[None, :])
    gam = np.tril(gam)
    return np.exp(ell), gam


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


def chunk_scan(variant, q, k, v, C, beta=None, a=None, r=None, qn=0.0, S0=None, P0=None, p0=None):
    """One head: q, k [L, dk], v [L, dv]; scalars [L].  Returns o, m, S and P or p."""
    L, dk = k.shape
    dv = v.shape[1]
    a = np.ones(L) if a is None else np.asarray(a, float)
    qn = np.broadcast_to(np.asarray(qn, float), (L,))
    S = np.zeros((dk, dv)) if S0 is None else np.array(S0, float)
    P = np.eye(dk) if P0 is None else np.array(P0, float)
    p = np.ones(dk) if p0 is None else np.array(p0, float)
    o = np.zeros((L, dv))
    m = np.zeros(L)
    for c0 in range(0, L, C):
        sl = slice(c0, min(c0 + C, L))
        Kc, Qc, Vc, ac = k[sl], q[sl], v[sl], a[sl]
        n = Kc.shape[0]
        A, gam = _gates(ac)
        if variant == "delta":
            Gm = beta[sl, None] * Kc
        elif variant == "kalman_diag":
            Gm = np.zeros((n, dk))
            for i in range(n):
                pp = ac[i] ** 2 * p + qn[sl][i]
                s = pp @ (Kc[i] ** 2) + r[sl][i]
                Gm[i] = pp * Kc[i] / s
                p = pp * r[sl][i] / (r[sl][i] + pp * Kc[i] ** 2)
        elif variant == "kalman_full":
            gamma = np.zeros(n)
            g_prev = 0.0
            for i in range(n):
                g_prev = ac[i] ** 2 * g_prev + qn[sl][i]
                gamma[i] = g_prev
            Bt = (A ** 2)[:, None] * (Kc @ P) + gamma[:, None] * Kc  # rows Pi_j k_j (P symmetric)
            G = np.tril((Kc @ Bt.T) * gam)
            G = G + np.tril(G, -1).T + np.diag(r[sl])
            Lf, D = _ldl(G)
            Z = (np.linalg.inv(Lf) * gam) @ Bt
            Gm = Z / D[:, None]
            w = (A[-1] / A) ** 2 * D
            P = (A[-1] ** 2) * P + gamma[-1] * np.eye(dk) - (Gm.T * w) @ Gm
            P = 0.5 * (P + P.T)
        else:
            raise ValueError(variant)
        N = np.tril((Kc @ Gm.T) * gam, -1)
        R = Vc - A[:, None] * (Kc @ S)
        E = np.linalg.solve(np.eye(n) + N, R)
        o[sl] = A[:, None] * (Qc @ S) + ((Qc @ Gm.T) * gam) @ E
        S = A[-1] * S + Gm.T @ ((A[-1] / A)[:, None] * E)
        m[sl] = np.linalg.norm(Gm, axis=1) * np.linalg.norm(E, axis=1)
    out = {"o": o, "m": m, "S": S}
    if variant == "kalman_full":
        out["P"] = P
    if variant == "kalman_diag":
        out["p"] = p
    return out
