"""The chunked backward model of the gated delta rule against the token-by-token backward oracle (CPU)."""

import numpy as np
import pytest

from chunk_model_backward import chunk_delta_backward
from oracle.backward import scan_delta_backward


@pytest.mark.parametrize("C", [1, 4, 16, 64])
@pytest.mark.parametrize("L", [37, 128])
def test_chunked_backward_equals_token_backward(C, L):
    rng = np.random.default_rng(C * 1000 + L)
    dk, dv = 6, 5
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    q, k = unit(rng.standard_normal((L, dk))), unit(rng.standard_normal((L, dk)))
    v = rng.standard_normal((L, dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(L)))
    a = np.exp(-np.log1p(np.exp(rng.standard_normal(L) - 2.0)))
    S0 = 0.3 * rng.standard_normal((dk, dv))
    dO, dm, dSL = rng.standard_normal((L, dv)), rng.standard_normal(L), rng.standard_normal((dk, dv))
    ref = scan_delta_backward(q, k, v, beta, dO, a=a, S0=S0, dm=dm, dS_L=dSL)
    got = chunk_delta_backward(q, k, v, beta, a, C, dO, S0=S0, dm=dm, dS_L=dSL)
    for key in ("dq", "dk", "dv", "dbeta", "da", "dS0"):
        scale = max(np.abs(ref[key]).max(), 1e-12)
        assert np.abs(got[key] - ref[key]).max() <= 1e-9 * scale, (key, np.abs(got[key] - ref[key]).max(), scale)


@pytest.mark.parametrize("C", [1, 8, 64])
def test_chunked_diagonal_backward_equals_token_backward(C):
    from chunk_model_backward import chunk_diag_backward
    from oracle.backward import scan_kalman_diag_backward
    rng = np.random.default_rng(C + 77)
    L, dk, dv = 70, 5, 4
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    q, k = unit(rng.standard_normal((L, dk))), unit(rng.standard_normal((L, dk)))
    v = rng.standard_normal((L, dv))
    r = np.log1p(np.exp(rng.standard_normal(L))) + 0.1
    a = np.exp(-np.log1p(np.exp(rng.standard_normal(L) - 2.0)))
    qn = np.full(L, 1e-3)
    S0, p0 = 0.3 * rng.standard_normal((dk, dv)), 0.5 + rng.random(dk)
    dO, dm = rng.standard_normal((L, dv)), rng.standard_normal(L)
    dSL, dpL = rng.standard_normal((dk, dv)), rng.standard_normal(dk)
    ref = scan_kalman_diag_backward(q, k, v, r, dO, a=a, qn=qn, S0=S0, p0=p0, dm=dm, dS_L=dSL, dp_L=dpL)
    got = chunk_diag_backward(q, k, v, r, a, qn, C, dO, S0=S0, p0=p0, dm=dm, dS_L=dSL, dp_L=dpL)
    for key in ("dq", "dk", "dv", "dr", "da", "dqn", "dS0", "dp0"):
        scale = max(np.abs(ref[key]).max(), 1e-12)
        assert np.abs(got[key] - ref[key]).max() <= 1e-9 * scale, (key, np.abs(got[key] - ref[key]).max(), scale)


@pytest.mark.parametrize("C", [1, 16, 64])
def test_chunked_isotropic_backward_equals_token_backward(C):
    from chunk_model_backward import chunk_iso_backward
    from oracle.backward import scan_kalman_iso_backward
    rng = np.random.default_rng(C + 99)
    L, dk, dv = 75, 5, 4
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    q, k = unit(rng.standard_normal((L, dk))), unit(rng.standard_normal((L, dk)))
    v = rng.standard_normal((L, dv))
    r = np.log1p(np.exp(rng.standard_normal(L))) + 0.1
    a = np.exp(-np.log1p(np.exp(rng.standard_normal(L) - 2.0)))
    qn = np.full(L, 1e-3)
    S0 = 0.3 * rng.standard_normal((dk, dv))
    dO, dm, dSL = rng.standard_normal((L, dv)), rng.standard_normal(L), rng.standard_normal((dk, dv))
    ref = scan_kalman_iso_backward(q, k, v, r, dO, a=a, qn=qn, S0=S0, c0=0.8, dm=dm, dS_L=dSL, dc_L=0.3)
    got = chunk_iso_backward(q, k, v, r, a, qn, C, dO, S0=S0, c0=0.8, dm=dm, dS_L=dSL, dc_L=0.3)
    for key in ("dq", "dk", "dv", "dr", "da", "dqn", "dS0", "dc0"):
        scale = max(np.abs(ref[key]).max(), 1e-12)
        assert np.abs(got[key] - ref[key]).max() <= 1e-9 * scale, (key, np.abs(got[key] - ref[key]).max(), scale)


def test_ldl_adjoint_matches_central_differences():
    from chunk_model_backward import _ldl, ldl_backward
    rng = np.random.default_rng(5)
    n = 6
    B = rng.standard_normal((n, n))
    G = B @ B.T + n * np.eye(n)
    dL, dD = np.tril(rng.standard_normal((n, n)), -1), rng.standard_normal(n)
    got = ldl_backward(*_ldl(G), dL, dD)
    h = 1e-6
    for i in range(n):
        for j in range(i + 1):
            E = np.zeros((n, n))
            E[i, j] = E[j, i] = 1.0  # the lower entry (i, j) stands for both mirror images
            Lp, Dp = _ldl(G + h * E)
            Lm, Dm = _ldl(G - h * E)
            num = (np.sum(dL * (Lp - Lm)) + np.sum(dD * (Dp - Dm))) / (2 * h)
            assert abs(got[i, j] - num) <= 1e-7 * max(1.0, abs(num)), (i, j, got[i, j], num)


@pytest.mark.parametrize("C", [1, 8, 64])
def test_chunked_full_backward_equals_token_backward(C):
    from chunk_model_backward import chunk_full_backward
    from oracle.backward import scan_kalman_full_backward
    rng = np.random.default_rng(C + 123)
    L, dk, dv = 70, 5, 4
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    q, k = unit(rng.standard_normal((L, dk))), unit(rng.standard_normal((L, dk)))
    v = rng.standard_normal((L, dv))
    r = np.log1p(np.exp(rng.standard_normal(L))) + 0.1
    a = np.exp(-np.log1p(np.exp(rng.standard_normal(L) - 3.0)))
    qn = np.full(L, 1e-3)
    B = rng.standard_normal((dk, dk)) / dk
    S0, P0 = 0.3 * rng.standard_normal((dk, dv)), 0.5 * np.eye(dk) + B @ B.T
    dO, dm, dSL = rng.standard_normal((L, dv)), rng.standard_normal(L), rng.standard_normal((dk, dv))
    X = rng.standard_normal((dk, dk))
    dPL = X + X.T
    ref = scan_kalman_full_backward(q, k, v, r, dO, a=a, qn=qn, S0=S0, P0=P0, dm=dm, dS_L=dSL, dP_L=dPL)
    ref["dP0"] = 0.5 * (ref["dP0"] + ref["dP0"].T)
    got = chunk_full_backward(q, k, v, r, a, qn, C, dO, S0=S0, P0=P0, dm=dm, dS_L=dSL, dP_L=dPL)
    for key in ("dq", "dk", "dv", "dr", "da", "dqn", "dS0", "dP0"):
        scale = max(np.abs(ref[key]).max(), 1e-12)
        assert np.abs(got[key] - ref[key]).max() <= 1e-8 * scale, (key, np.abs(got[key] - ref[key]).max(), scale)


@pytest.mark.parametrize("block", [1, 5, 64])
def test_full_cov_backward_tokens_with_memory_step_equals_token_backward(block):
    """The covariance side the full-Kalman backward kernels run (carried M = Pb + Pb^T, blocks recomputed
    from checkpoints), fed with the oracle's memory step for dg, gives the oracle's gradients."""
    from chunk_model_backward import full_cov_backward_tokens
    from oracle.backward import _memory_step_backward, scan_kalman_full_backward
    rng = np.random.default_rng(block + 7)
    L, dk, dv = 23, 6, 4
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    q, k = unit(rng.standard_normal((L, dk))), unit(rng.standard_normal((L, dk)))
    v = rng.standard_normal((L, dv))
    r = np.log1p(np.exp(rng.standard_normal(L))) + 0.1
    a = np.exp(-np.log1p(np.exp(rng.standard_normal(L) - 3.0)))
    a[4] = 0.0
    qn = 1e-3 + 1e-2 * rng.random(L)
    B = rng.standard_normal((dk, dk)) / dk
    S0, P0 = 0.3 * rng.standard_normal((dk, dv)), 0.5 * np.eye(dk) + B @ B.T
    dO, dm, dSL = rng.standard_normal((L, dv)), rng.standard_normal(L), rng.standard_normal((dk, dv))
    dPL = rng.standard_normal((dk, dk))  # not symmetric: the carried M symmetrises it
    ref = scan_kalman_full_backward(q, k, v, r, dO, a=a, qn=qn, S0=S0, P0=P0, dm=dm, dS_L=dSL, dP_L=dPL)
    # forward, then the memory backward with the gains as given inputs (its dg feeds the covariance side)
    S, P, states, gains, res = S0.copy(), P0.copy(), [S0.copy()], [], []
    for t in range(L):
        Pm = a[t] ** 2 * P + qn[t] * np.eye(dk)
        u = Pm @ k[t]
        s = k[t] @ u + r[t]
        g = u / s
        P = Pm - np.outer(u, u) / s
        e = v[t] - a[t] * S.T @ k[t]
        S = a[t] * S + np.outer(g, e)
        states.append(S.copy()), gains.append(g), res.append(e)
    G = dSL[None].copy()
    dg = np.zeros((L, dk))
    mem = {key: np.zeros(shape) for key, shape in (("dq", (L, dk)), ("dk", (L, dk)), ("dv", (L, dv)), ("da", L))}
    for t in range(L - 1, -1, -1):
        G, dq, de, dkt, da_t, dgt = _memory_step_backward(G, gains[t][None], res[t][None], k[t][None], q[t][None],
                                                         states[t + 1][None], states[t][None], a[t:t + 1],
                                                         dO[t][None], dm[t:t + 1])
        mem["dq"][t], mem["dk"][t], mem["dv"][t], mem["da"][t], dg[t] = dq[0], dkt[0], de[0], da_t[0], dgt[0]
    cov = full_cov_backward_tokens(k, r, a, qn, P0, dg, dP_L=dPL, block=block)
    got = {"dq": mem["dq"], "dv": mem["dv"], "dk": mem["dk"] + cov["dk"], "da": mem["da"] + cov["da"],
           "dr": cov["dr"], "dqn": cov["dqn"], "dS0": G[0], "dP0": cov["dP0"]}
    ref["dP0"] = 0.5 * (ref["dP0"] + ref["dP0"].T)
    for key in ("dq", "dk", "dv", "dr", "da", "dqn", "dS0", "dP0"):
        scale = max(np.abs(ref[key]).max(), 1e-12)
        assert np.abs(got[key] - ref[key]).max() <= 1e-9 * scale, (key, np.abs(got[key] - ref[key]).max(), scale)
