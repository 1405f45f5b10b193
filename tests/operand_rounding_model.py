"""Float64 model of the chunk kernel's operand roundings (d = 64 and 128).

Test infrastructure: it repeats the chunk form of the scan (the generalised
WY form: (I + N) E = V - diag(A) K S0, O = diag(A) Q S0 + AT R, S_C = A_C S0 +
G^T diag(A_C / A_j) E) in float64, rounding every tensor-core operand the way
the kernel does before each product, so that the error those roundings cost at
layer length can be measured on the CPU against the exact scan.  It shares no
code with the oracle or the kernels.

Roundings: ``exact`` (none); ``f16`` (one fp16 value, round to nearest, with
fp16's range and subnormals: what the kernel does now, except that the Kalman
gains enter K G^T and Q G^T as an fp16 hi + lo pair); ``bf16_pair`` (bf16 hi
+ bf16 lo, about 16 significand bits).
"""

import numpy as np
import torch


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).double().numpy()


ROUNDINGS = {
    "exact": lambda x: np.asarray(x, np.float64),
    "f16": lambda x: np.asarray(x, np.float64).astype(np.float16).astype(np.float64),
    "bf16_pair": lambda x: _bf16(x) + _bf16(np.asarray(x) - _bf16(x)),
}


def chunk_scan_rounded(variant, q, k, v, beta, a, r, qn, rounding, C=64):
    """One head (q, k [L, d_k], v [L, d_v], scalars [L]); returns o, m, S."""
    rnd = ROUNDINGS[rounding]
    L, dk = k.shape
    S = np.zeros((dk, v.shape[1]))
    p = np.ones(dk)
    o = np.zeros((L, v.shape[1]))
    m = np.zeros(L)
    for c0 in range(0, L, C):
        sl = slice(c0, min(c0 + C, L))
        K, Q, V, ac = k[sl], q[sl], v[sl], a[sl]
        n = K.shape[0]
        ell = np.cumsum(np.log(np.maximum(ac, np.exp(-60.0))))
        A = np.exp(ell)
        gam = np.tril(np.exp(ell[:, None] - ell[None, :]))
        if variant == "delta":
            G = beta[sl, None] * K
            Gr = K  # the kernel multiplies by K itself and carries beta in fp32 scalars
            bscale = beta[sl]
        else:
            G = np.zeros((n, dk))
            for i in range(n):
                pp = ac[i] ** 2 * p + qn
                G[i] = pp * K[i] / (pp @ K[i] ** 2 + r[sl][i])
                p = pp * r[sl][i] / (r[sl][i] + pp * K[i] ** 2)
            Gr = rnd(G)
            bscale = np.ones(n)
        # the gains in K G^T and Q G^T: the fp16 pair under f16, else as in the state product
        Gd = Gr + rnd(G - Gr) if rounding == "f16" and variant != "delta" else Gr
        Kr, Qr = rnd(K), rnd(Q)
        N = np.tril((Kr @ Gd.T) * gam * bscale[None, :], -1)
        T = np.linalg.inv(np.eye(n) + N)
        Att = np.tril((Qr @ Gd.T) * gam * bscale[None, :])
        Tr = rnd(T)
        AT = Att @ Tr
        Sr = rnd(S)
        R = V - A[:, None] * (Kr @ Sr)
        Rr = rnd(R)
        E = Tr @ Rr
        o[sl] = A[:, None] * (Qr @ Sr) + rnd(AT) @ Rr
        S = A[-1] * S + Gr.T @ rnd((A[-1] / A * bscale)[:, None] * E)
        m[sl] = np.linalg.norm(G, axis=1) * np.linalg.norm(E, axis=1)
    return o, m, S
