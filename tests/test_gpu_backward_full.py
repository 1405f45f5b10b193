"""GPU parity of the full-covariance Kalman backward (kdn_scan_kalman_full_backward) with the float64 adjoint oracle.

The oracle (oracle/backward.py) runs the token recurrence backwards with every state and covariance kept; the
CUDA path runs the covariance chain forward (gains, P at every 64-token block start), the memory backward with
the gains as inputs, and the covariance chain backwards with each block recomputed from its checkpoint.  Every
gradient is compared per head with the normwise metric of the forward tests (1e-4 for fp32 inputs, 3e-3 for
bf16 inputs).  dP0 is the gradient for a symmetric P0 (the forward requires a symmetric covariance), so it is
compared with the symmetric part of the oracle's entrywise dP0.  Cases: several blocks with a ragged tail, per-
token and scalar process noise, zero gates, a non-zero start state and a general symmetric PD P0, the surprise,
final-state and (non-symmetric) final-covariance upstream gradients, unequal d_k / d_v, an empty sequence, and
the layer shape at full size on a sampled head.
"""

import numpy as np
import pytest
import torch

from delta_rule_recurrent_scan_b200 import kdn
from delta_rule_recurrent_scan_b200.workloads import WORKLOADS, make_scan_inputs
from oracle.backward import scan_kalman_full_backward as oracle_full_backward
from parity import TOL, normwise_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
KEYS = ("dq", "dk", "dv", "dr", "da", "dqn", "dS0", "dP0")


def _np(t):
    return None if t is None else t.detach().double().cpu().numpy()


def _upstream(B, H, L, dk, dv, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    dO = torch.randn(B, H, L, dv, device=DEV, generator=g)
    dm = torch.randn(B, H, L, device=DEV, generator=g)
    dS_L = torch.randn(B, H, dk, dv, device=DEV, generator=g) * 0.1
    S0 = torch.randn(B, H, dk, dv, device=DEV, generator=g) * 0.1
    X = torch.randn(B, H, dk, dk, device=DEV, generator=g) / dk ** 0.5
    P0 = 0.5 * torch.eye(dk, device=DEV) + X @ X.transpose(-1, -2)
    dP_L = torch.randn(B, H, dk, dk, device=DEV, generator=g) * 0.1
    return dO, dm, dS_L, S0, P0, dP_L


def _check(x, qn, dO, dm, dS_L, S0, P0, dP_L, tol, heads=None):
    got = kdn.scan_kalman_full_backward(x["q"], x["k"], x["v"], x["r"], dO, a=x["a"], qn=qn, S0=S0, P0=P0, dm=dm,
                                        dS_L=dS_L, dP_L=dP_L)
    torch.cuda.synchronize()

    def pick(t):
        if t is None or isinstance(t, float):
            return t
        if heads is None:
            return _np(t)
        return np.stack([_np(t[b, h]) for b, h in heads])[None]

    ref = oracle_full_backward(pick(x["q"]), pick(x["k"]), pick(x["v"]), pick(x["r"]), pick(dO), a=pick(x["a"]),
                               qn=pick(qn), S0=pick(S0), P0=pick(P0), dm=pick(dm), dS_L=pick(dS_L),
                               dP_L=pick(dP_L))
    ref["dP0"] = 0.5 * (ref["dP0"] + np.swapaxes(ref["dP0"], -1, -2))
    errs = {}
    for key in KEYS:
        g = got[key]
        if heads is not None:
            g = torch.stack([g[b, h] for b, h in heads])[None]
        assert torch.isfinite(g).all(), key
        errs[key] = normwise_err(g, ref[key], lead=2)
    bad = {k_: e for k_, e in errs.items() if not e <= tol}
    assert not bad, f"errors above {tol}: {errs}"
    return errs


@pytest.mark.parametrize("d,L", [(64, 150), (128, 100), (32, 77), (16, 33)])
def test_full_backward_reduced_shapes_bf16(d, L):
    w = WORKLOADS["kalman_full_d128"].with_(dk=d, dv=d)
    x = make_scan_inputs(w, seed=61, device=DEV, B=1, H=2, L=L)
    dO, dm, dS_L, S0, P0, dP_L = _upstream(1, 2, L, d, d, seed=62)
    _check(x, x["qn"], dO, dm, dS_L, S0, P0, dP_L, TOL["bf16"])


@pytest.mark.parametrize("dk,dv", [(16, 16), (64, 32), (32, 128)])
def test_full_backward_fp32_inputs_per_token_noise_and_unequal_dims(dk, dv):
    w = WORKLOADS["kalman_full_d128"].with_(dtype="f32", dk=dk, dv=dv)
    x = make_scan_inputs(w, seed=63, device=DEV, B=2, H=1, L=70)
    qn = 1e-3 + 1e-2 * torch.rand(2, 1, 70, device=DEV)
    dO, dm, dS_L, S0, P0, dP_L = _upstream(2, 1, 70, dk, dv, seed=64)
    _check(x, qn, dO, dm, dS_L, S0, P0, dP_L, TOL["f32"])


def test_full_backward_resets_and_no_optional_inputs():
    """Zero gates (the covariance restarts from Qn I, the memory from zero), and a call with only dO."""
    w = WORKLOADS["kalman_full_d128"].with_(dk=64, dv=64)
    x = make_scan_inputs(w, seed=65, device=DEV, B=2, H=2, L=130)
    x["a"][:, :, ::7] = 0.0
    x["a"][:, :, 3::11] = 1.0
    dO, dm, dS_L, S0, P0, dP_L = _upstream(2, 2, 130, 64, 64, seed=66)
    _check(x, x["qn"], dO, dm, dS_L, S0, P0, dP_L, TOL["bf16"])
    _check(x, x["qn"], dO, None, None, None, None, None, TOL["bf16"])


def test_full_backward_empty_sequence_passes_the_final_gradients_through():
    w = WORKLOADS["kalman_full_d128"].with_(dk=64, dv=64)
    x = make_scan_inputs(w, seed=67, device=DEV, B=1, H=2, L=0)
    dS_L = torch.randn(1, 2, 64, 64, device=DEV)
    dP_L = torch.randn(1, 2, 64, 64, device=DEV)
    got = kdn.scan_kalman_full_backward(x["q"], x["k"], x["v"], x["r"], torch.empty(1, 2, 0, 64, device=DEV),
                                        a=x["a"], qn=x["qn"], dS_L=dS_L, dP_L=dP_L)
    torch.cuda.synchronize()
    assert torch.equal(got["dS0"], dS_L)
    assert torch.allclose(got["dP0"], 0.5 * (dP_L + dP_L.transpose(-1, -2)), rtol=0, atol=1e-6)


def test_full_backward_full_layer_sampled_head():
    """The full-Kalman layer (B2 H8 L4096, d=128) at full size, checked on a sampled head."""
    w = WORKLOADS["kalman_full_d128"]
    x = make_scan_inputs(w, seed=0, device=DEV)
    dO, dm, _, _, _, _ = _upstream(w.B, w.H, w.L, w.dk, w.dv, seed=68)
    _check(x, x["qn"], dO, dm, None, None, None, None, TOL["bf16"], heads=[(1, 5)])
