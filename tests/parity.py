"""Helpers shared by the GPU parity tests: run the CUDA path and the oracle on
the same seeded inputs and compare them with the normwise per-head metric.

Error metric (one reading of "max relative error"): for each head (b, h),
max |x - y| / max |y| over that head's elements; the test takes the max over
heads.  Elementwise relative error is undefined near the zeros of o.
"""

import numpy as np
import torch

import oracle
from delta_rule_recurrent_scan_b200 import kdn

TOL = {"f32": 1e-4, "bf16": 3e-3}

# Two CUDA runs of the same scan against each other (two chunkings, segments against the serial scan,
# decode against the scan).  Paths built from fp32 CUDA-core arithmetic agree to 1e-4.  The chunk kernel
# (bf16 inputs, d = 64 and 128) rounds its tensor-core operands to fp16 once (unit roundoff 2^-11 =
# 4.9e-4; a float64 emulation of its roundings over 8192-token layers stays below 6e-4 against the exact
# scan), so two runs that each carry such roundings differ by up to about twice that.
SELF_TOL = 1e-4
SELF_TOL_F16 = 1.5e-3


def self_tol(d):
    """Agreement expected between two CUDA runs of the bf16 chunk path at head dimension d (d_k = d_v)."""
    return SELF_TOL_F16 if d in (64, 128) else SELF_TOL


def normwise_err(x, y, lead=2):
    x = torch.as_tensor(x).double().cpu()
    y = torch.as_tensor(y).double().cpu()
    n = int(np.prod(x.shape[:lead]))
    x, y = x.reshape(n, -1), y.reshape(n, -1)
    den = y.abs().amax(dim=1).clamp_min(1e-30)
    return float(((x - y).abs().amax(dim=1) / den).max())


def initial_state(variant, B, H, dk, dv, device):
    S = torch.zeros(B, H, dk, dv, dtype=torch.float32, device=device)
    if variant == "kalman_full":
        return S, torch.eye(dk, dtype=torch.float32, device=device).repeat(B, H, 1, 1)
    if variant == "kalman_diag":
        return S, torch.ones(B, H, dk, dtype=torch.float32, device=device)
    if variant == "kalman_iso":
        return S, torch.ones(B, H, dtype=torch.float32, device=device)
    return S, None


def run_gpu(variant, x, S=None, C=None, chunk=0, out_dtype=None):
    q, k, v = x["q"], x["k"], x["v"]
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    if S is None:
        S, C = initial_state(variant, B, H, dk, dv, q.device)
    if variant == "delta":
        o, m, S = kdn.scan_delta(q, k, v, x["beta"], a=x["a"], S=S, chunk=chunk, out_dtype=out_dtype)
        return {"o": o, "m": m, "S": S}
    fn = {"kalman_full": kdn.scan_kalman_full, "kalman_diag": kdn.scan_kalman_diag,
          "kalman_iso": kdn.scan_kalman_iso}[variant]
    key = {"kalman_full": "P", "kalman_diag": "p", "kalman_iso": "c"}[variant]
    kw = {key: C}
    o, m, S, C = fn(q, k, v, x["r"], a=x["a"], qn=x["qn"], S=S, chunk=chunk, out_dtype=out_dtype, **kw)
    return {"o": o, "m": m, "S": S, key: C}


def _np(t):
    return None if t is None else t.detach().double().cpu().numpy()


def run_oracle(variant, x, S0=None, C0=None, heads=None):
    """Oracle on the same inputs; ``heads`` = list of (b, h) to restrict to."""
    def pick(t):
        if t is None:
            return None
        if heads is None:
            return _np(t)
        return np.stack([_np(t[b, h]) for b, h in heads])[None]

    q, k, v = pick(x["q"]), pick(x["k"]), pick(x["v"])
    a = pick(x["a"])
    if variant == "delta":
        return oracle.scan_delta(q, k, v, pick(x["beta"]), a=a, S0=pick(S0))
    if variant == "kalman_full":
        return oracle.scan_kalman_full(q, k, v, r=pick(x["r"]), a=a, qn=x["qn"], S0=pick(S0), P0=pick(C0))
    if variant == "kalman_iso":
        return oracle.scan_kalman_iso(q, k, v, r=pick(x["r"]), a=a, qn=x["qn"], S0=pick(S0), c0=pick(C0))
    return oracle.scan_kalman_diag(q, k, v, r=pick(x["r"]), a=a, qn=x["qn"], S0=pick(S0), p0=pick(C0))


BF16_HALF_ULP = 2.0 ** -8  # bf16 keeps 8 significand bits: round-to-nearest costs up to 2^-8 relative


def normwise_err_rounded(x, y, lead=2):
    """Normwise error after removing what rounding y to bf16 alone may cost:
    max over heads of max(|x - y| - 2^-8 |y|, 0) / max |y|."""
    x = torch.as_tensor(x).double().cpu()
    y = torch.as_tensor(y).double().cpu()
    n = int(np.prod(x.shape[:lead]))
    x, y = x.reshape(n, -1), y.reshape(n, -1)
    den = y.abs().amax(dim=1).clamp_min(1e-30)
    excess = ((x - y).abs() - BF16_HALF_ULP * y.abs()).clamp_min(0.0)
    return float((excess.amax(dim=1) / den).max())


def compare(got, ref, tol, heads=None):
    """Max normwise error over the outputs; returns a dict key -> error.  A bf16
    output is held to the tolerance beyond its own rounding (2^-8 of each element)."""
    errs = {}
    for key, val in ref.items():
        if key not in got:
            continue
        g = got[key]
        if heads is not None:
            g = torch.stack([g[b, h] for b, h in heads])[None]
        if g.dtype == torch.bfloat16:
            errs[key] = normwise_err_rounded(g, val)
        else:
            errs[key] = normwise_err(g, val)
    bad = {k_: e for k_, e in errs.items() if not (e <= tol)}
    assert not bad, f"errors above {tol}: {errs}"
    return errs


def assert_symmetric_pd(P, tol=TOL["bf16"]):
    """Every head's returned covariance is symmetric to ``tol`` (normwise) and positive definite
    (a float64 Cholesky of its symmetric part succeeds)."""
    P = P.detach().double().cpu().reshape(-1, P.shape[-2], P.shape[-1])
    asym = (P - P.transpose(1, 2)).flatten(1).abs().amax(1) / P.flatten(1).abs().amax(1)
    assert float(asym.max()) <= tol, float(asym.max())
    _, info = torch.linalg.cholesky_ex(0.5 * (P + P.transpose(1, 2)))
    assert int(info.abs().max()) == 0, "P is not positive definite"
