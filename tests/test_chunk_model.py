"""The chunked forms the kernels compute equal the token-by-token oracle (float64)."""

import numpy as np
import pytest

from chunk_model import chunk_scan
from oracle import scan_delta, scan_kalman_diag, scan_kalman_full


def _inputs(seed, L, dk, dv, zero_gates=False):
    rng = np.random.default_rng(seed)
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)  # noqa: E731
    q = unit(rng.standard_normal((L, dk)))
    k = unit(rng.standard_normal((L, dk)))
    v = rng.standard_normal((L, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal(L)))
    a = np.exp(-np.log1p(np.exp(rng.standard_normal(L) - 2.0)))
    if zero_gates:
        a[rng.integers(0, L, 4)] = 0.0
    r = np.log1p(np.exp(rng.standard_normal(L))) + 0.1
    S0 = 0.3 * rng.standard_normal((dk, dv))
    M = rng.standard_normal((dk, dk))
    P0 = M @ M.T / dk + 0.5 * np.eye(dk)
    p0 = 0.5 + rng.random(dk)
    return q, k, v, beta, a, r, S0, P0, p0


@pytest.mark.parametrize("C", [1, 4, 16, 64])
@pytest.mark.parametrize("variant", ["delta", "kalman_diag", "kalman_full"])
@pytest.mark.parametrize("zero_gates", [False, True])
def test_chunk_forms_equal_oracle(C, variant, zero_gates):
    L, dk, dv = 100, 12, 7
    q, k, v, beta, a, r, S0, P0, p0 = _inputs(C + 7 * zero_gates, L, dk, dv, zero_gates)
    qn = 1e-3
    if variant == "delta":
        ref = scan_delta(q[None], k[None], v[None], beta[None], a=a[None], S0=S0[None])
        got = chunk_scan(variant, q, k, v, C, beta=beta, a=a, S0=S0)
    elif variant == "kalman_diag":
        ref = scan_kalman_diag(q[None], k[None], v[None], r=r[None], a=a[None], qn=qn, S0=S0[None], p0=p0[None])
        got = chunk_scan(variant, q, k, v, C, a=a, r=r, qn=qn, S0=S0, p0=p0)
    else:
        ref = scan_kalman_full(q[None], k[None], v[None], r=r[None], a=a[None], qn=qn, S0=S0[None], P0=P0[None])
        got = chunk_scan(variant, q, k, v, C, a=a, r=r, qn=qn, S0=S0, P0=P0)
    for key in got:
        np.testing.assert_allclose(got[key], ref[key][0], rtol=1e-8, atol=1e-10, err_msg=key)
