"""GPU parity of the segment-parallel scans (several CTAs per head, chained segment maps).

Each case runs the CUDA path with an explicit or library-chosen segment count and compares it with the
float64 oracle (normwise per head, 3e-3 for bf16 inputs) and with the serial CUDA scan (segments = 1).
Segments that are not a whole number of 64-token chunks, start states other than zero and the
library's own choice at the layer sizes where it applies are all covered.
"""

import ctypes

import pytest
import torch

from delta_rule_recurrent_scan_b200 import kdn
from delta_rule_recurrent_scan_b200.workloads import WORKLOADS, make_scan_inputs
from parity import TOL, assert_symmetric_pd, compare, initial_state, run_oracle, self_tol

pytestmark = pytest.mark.gpu
DEV = "cuda"
KEY = {"kalman_full": "P", "kalman_diag": "p", "kalman_iso": "c"}


def _run(variant, x, S, C, segments, out_dtype=None, workspace=None):
    q, k, v = x["q"], x["k"], x["v"]
    if variant == "delta":
        o, m, S = kdn.scan_delta(q, k, v, x["beta"], a=x["a"], S=S, segments=segments, out_dtype=out_dtype,
                                 workspace=workspace)
        return {"o": o, "m": m, "S": S}
    fn = {"kalman_full": kdn.scan_kalman_full, "kalman_diag": kdn.scan_kalman_diag,
          "kalman_iso": kdn.scan_kalman_iso}[variant]
    o, m, S, C = fn(q, k, v, x["r"], a=x["a"], qn=x["qn"], S=S, segments=segments, out_dtype=out_dtype,
                    workspace=workspace, **{KEY[variant]: C})
    return {"o": o, "m": m, "S": S, KEY[variant]: C}


def _start(variant, B, H, d, seed):
    """A non-trivial start: S0 ~ N(0, 1/d), p0 in [0.5, 1.5], c0 in [0.5, 1.5], P0 = I/2 + a small SPD part."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    S = (torch.randn(B, H, d, d, generator=g) / d ** 0.5).to(DEV)
    if variant == "delta":
        return S, None
    if variant == "kalman_diag":
        return S, (0.5 + torch.rand(B, H, d, generator=g)).to(DEV)
    if variant == "kalman_iso":
        return S, (0.5 + torch.rand(B, H, generator=g)).to(DEV)
    A = torch.randn(B, H, d, d, generator=g) / d
    return S, (0.5 * torch.eye(d) + A @ A.transpose(-1, -2)).to(DEV)


def _clone(S, C):
    return S.clone(), None if C is None else C.clone()


def _check(variant, x, segments, S0=None, C0=None, out_dtype=None):
    B, H, L, d = x["q"].shape
    if S0 is None:
        S0, C0 = initial_state(variant, B, H, d, d, DEV)
    got = _run(variant, x, *_clone(S0, C0), segments, out_dtype=out_dtype)
    ser = _run(variant, x, *_clone(S0, C0), 1, out_dtype=out_dtype)
    torch.cuda.synchronize()
    compare(got, run_oracle(variant, x, S0=S0, C0=C0), TOL["bf16"])
    compare(got, {k_: v_.double().cpu() for k_, v_ in ser.items()}, self_tol(d) if out_dtype is None else 1e-2)
    return got


VARIANTS = ["delta", "kalman_diag", "kalman_iso", "kalman_full"]


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("d", [64, 128])
def test_library_choice_splits_few_heads(variant, d):
    """B*H = 2 and L = 1024: the library picks 8 segments of two chunks each."""
    w = WORKLOADS["gdn_d128"].with_(variant=variant, dk=d, dv=d, qn=1e-3)
    x = make_scan_inputs(w, seed=11, device=DEV, B=1, H=2, L=1024)
    n = kdn.plan(variant, 1, 2, 1024, d, d)["launches"]
    assert n >= (4 if d == 64 else 5), n  # the segment-parallel plan (one map run on [S | M] at d = 64)
    _check(variant, x, 0)


@pytest.mark.parametrize("variant", VARIANTS)
def test_ragged_segments_and_a_nonzero_start(variant):
    """Three segments of 150 tokens (two chunks and a 22-token tail each), from a random start state."""
    w = WORKLOADS["gdn_d128"].with_(variant=variant, qn=1e-3)
    x = make_scan_inputs(w, seed=12, device=DEV, B=2, H=1, L=450)
    S0, C0 = _start(variant, 2, 1, 128, seed=13)
    _check(variant, x, 3, S0, C0)


@pytest.mark.parametrize("variant", ["delta", "kalman_diag"])
def test_many_short_segments_and_bf16_output(variant):
    """32 segments of 64 tokens (one chunk each) over one head, bf16 o."""
    w = WORKLOADS["gdn_d64"].with_(variant=variant, qn=1e-3)
    x = make_scan_inputs(w, seed=14, device=DEV, B=1, H=1, L=2048)
    _check(variant, x, 32, out_dtype=torch.bfloat16)


def test_full_size_kalman_full_layer_uses_segments():
    """The full-covariance layer (B = 2, H = 8, L = 4096, d = 128) runs 8 segments per head; two sampled
    heads are checked against the oracle over the whole sequence."""
    w = WORKLOADS["kalman_full_d128"]
    assert kdn.plan("kalman_full", w.B, w.H, w.L, w.dk, w.dv)["launches"] == 9  # 3 of them build the chunk-start covariances
    x = make_scan_inputs(w, seed=0, device=DEV)
    S0, C0 = initial_state("kalman_full", w.B, w.H, w.dk, w.dv, DEV)
    got = _run("kalman_full", x, *_clone(S0, C0), 0)
    heads = [(0, 3), (1, 7)]
    ref = run_oracle("kalman_full", x, S0=S0, C0=C0, heads=heads)
    compare(got, ref, TOL["bf16"], heads=heads)
    assert_symmetric_pd(got["P"])


def test_segment_requests_are_validated():
    w = WORKLOADS["gdn_d128"]
    x = make_scan_inputs(w, seed=15, device=DEV, B=1, H=1, L=450)
    S0, _ = initial_state("delta", 1, 1, 128, 128, DEV)
    with pytest.raises(kdn.KdnError) as e:
        _run("delta", x, S0, None, 7)  # 7 does not divide 450
    assert e.value.status == kdn.KDN_ERR_INVALID_ARG
    with pytest.raises(kdn.KdnError) as e:
        _run("delta", x, S0, None, -1)
    assert e.value.status == kdn.KDN_ERR_INVALID_ARG
    # the serial workspace is too small for a segmented scan
    small = torch.empty(kdn.workspace_bytes("delta", 1, 1, 450, 128, 128, segments=1), dtype=torch.uint8, device=DEV)
    assert kdn.workspace_bytes("delta", 1, 1, 450, 128, 128, segments=3) > small.numel()
    with pytest.raises(kdn.KdnError) as e:
        _run("delta", x, S0, None, 3, workspace=small)
    assert e.value.status == kdn.KDN_ERR_INVALID_ARG


def test_many_heads_stay_serial():
    """At the layer sizes with 128 heads the library keeps one CTA per head."""
    for name in ("kalman_diag_d128", "gdn_d128", "kalman_iso_d128"):
        w = WORKLOADS[name]
        assert kdn.plan(w.variant, w.B, w.H, w.L, w.dk, w.dv)["launches"] == 1, name
