"""GPU parity of the gated delta rule backward (kdn_scan_delta_backward) with the float64 adjoint oracle.

The oracle (oracle/backward.py) runs the token recurrence backwards with every state kept; the CUDA
path re-runs the forward with 32-token checkpoints and walks the chunks backwards.  Every gradient is
compared per head with the normwise metric of the forward tests: 1e-4 for fp32 inputs, 3e-3 for bf16
inputs.  Cases: reduced shapes spanning several chunks with a ragged tail, zero gates (resets), beta in
{0, 1}, a non-zero start state, surprise and final-state upstream gradients, every supported head size
and unequal d_k / d_v; the layer shapes at full size on sampled heads.
"""

import numpy as np
import pytest
import torch

from delta_rule_recurrent_scan_b200 import kdn
from delta_rule_recurrent_scan_b200.workloads import WORKLOADS, make_scan_inputs
from oracle.backward import scan_delta_backward as oracle_backward
from parity import TOL, normwise_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
KEYS = ("dq", "dk", "dv", "dbeta", "da", "dS0")


def _upstream(B, H, L, dk, dv, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    dO = torch.randn(B, H, L, dv, device=DEV, generator=g)
    dm = torch.randn(B, H, L, device=DEV, generator=g)
    dS_L = torch.randn(B, H, dk, dv, device=DEV, generator=g) * 0.1
    S0 = torch.randn(B, H, dk, dv, device=DEV, generator=g) * 0.1
    return dO, dm, dS_L, S0


def _np(t):
    return None if t is None else t.detach().double().cpu().numpy()


def _check(x, dO, dm, dS_L, S0, tol, heads=None):
    got = kdn.scan_delta_backward(x["q"], x["k"], x["v"], x["beta"], dO, a=x["a"], S0=S0, dm=dm, dS_L=dS_L)
    torch.cuda.synchronize()

    def pick(t):
        if t is None:
            return None
        if heads is None:
            return _np(t)
        return np.stack([_np(t[b, h]) for b, h in heads])[None]

    ref = oracle_backward(pick(x["q"]), pick(x["k"]), pick(x["v"]), pick(x["beta"]), pick(dO), a=pick(x["a"]),
                          S0=pick(S0), dm=pick(dm), dS_L=pick(dS_L))
    errs = {}
    for key in KEYS:
        g = got[key]
        if heads is not None:
            g = torch.stack([g[b, h] for b, h in heads])[None]
        assert torch.isfinite(g).all(), key
        errs[key] = normwise_err(g, ref[key])
    bad = {k_: e for k_, e in errs.items() if not e <= tol}
    assert not bad, f"errors above {tol}: {errs}"
    return errs


@pytest.mark.parametrize("d,L", [(64, 150), (128, 100), (32, 77), (16, 33)])
def test_backward_reduced_shapes_bf16(d, L):
    w = WORKLOADS["gdn_d128"].with_(dk=d, dv=d)
    x = make_scan_inputs(w, seed=31, device=DEV, B=1, H=2, L=L)
    dO, dm, dS_L, S0 = _upstream(1, 2, L, d, d, seed=32)
    _check(x, dO, dm, dS_L, S0, TOL["bf16"])


@pytest.mark.parametrize("dk,dv", [(16, 16), (64, 32), (32, 128)])
def test_backward_fp32_inputs_and_unequal_dims(dk, dv):
    w = WORKLOADS["gdn_d64"].with_(dtype="f32", dk=dk, dv=dv)
    x = make_scan_inputs(w, seed=33, device=DEV, B=2, H=1, L=70)
    dO, dm, dS_L, S0 = _upstream(2, 1, 70, dk, dv, seed=34)
    _check(x, dO, dm, dS_L, S0, TOL["f32"])


def test_backward_resets_and_extreme_writes():
    w = WORKLOADS["gdn_d64"]
    x = make_scan_inputs(w, seed=35, device=DEV, B=2, H=2, L=130)
    x["a"][:, :, ::7] = 0.0   # full resets
    x["a"][:, :, 3::11] = 1.0
    x["beta"][:, :, 5::13] = 0.0
    x["beta"][:, :, 6::13] = 1.0
    dO, dm, dS_L, S0 = _upstream(2, 2, 130, 64, 64, seed=36)
    _check(x, dO, dm, dS_L, S0, TOL["bf16"])


def test_backward_without_optional_inputs():
    """No gate (a = 1; da is the gradient at 1), no surprise or final-state upstream, zero start state."""
    w = WORKLOADS["gdn_d64"].with_(a_shift=None)
    x = make_scan_inputs(w, seed=37, device=DEV, B=1, H=2, L=64)
    dO, _, _, _ = _upstream(1, 2, 64, 64, 64, seed=38)
    _check(x, dO, None, None, None, TOL["bf16"])


def test_backward_empty_sequence_passes_the_state_gradient_through():
    w = WORKLOADS["gdn_d64"]
    x = make_scan_inputs(w, seed=39, device=DEV, B=1, H=1, L=0)
    dS_L = torch.randn(1, 1, 64, 64, device=DEV)
    got = kdn.scan_delta_backward(x["q"], x["k"], x["v"], x["beta"], torch.empty(1, 1, 0, 64, device=DEV),
                                  a=x["a"], dS_L=dS_L)
    torch.cuda.synchronize()
    assert torch.equal(got["dS0"], dS_L)


@pytest.mark.parametrize("name", ["gdn_d64", "gdn_d128"])
def test_backward_full_layer_sampled_heads(name):
    """The layer shape at full size (the launch the benchmark times), checked on sampled heads."""
    w = WORKLOADS[name]
    x = make_scan_inputs(w, seed=0, device=DEV)
    dO, dm, _, _ = _upstream(w.B, w.H, w.L, w.dk, w.dv, seed=40)
    heads = [(0, 1)] if name == "gdn_d128" else [(0, 1), (w.B - 1, w.H - 2)]
    _check(x, dO, dm, None, None, TOL["bf16"], heads=heads)
