"""The allocation-free full-Kalman entry point (kdn_scan_kalman_full_noalloc).

It exists for callers that may not call cudaMalloc while running and have no
workspace to pass: its scratch is a static device array inside the library.
These tests call it through the C ABI and check it against the allocating
entry point (kdn_scan_kalman_full) on two calls in a row, the second one
continuing the state the first one left, so that a stale scratch between
calls would show.  This file is collected last on purpose.
"""

import ctypes

import pytest
import torch

from delta_rule_recurrent_scan_b200 import build, kdn
from delta_rule_recurrent_scan_b200.workloads import WORKLOADS, make_scan_inputs

TOL = 3e-3  # the bf16-input tolerance of the parity tests


def _err(x, y):
    x, y = x.double().flatten(1), y.double().flatten(1)
    return float(((x - y).abs().amax(1) / y.abs().amax(1).clamp_min(1e-30)).max())


def _noalloc_c_abi(x, S, P, o, m, segments=0):
    L = kdn.lib()
    B, H, T, dk = x["q"].shape
    d = kdn.Dims(B, H, T, dk, x["v"].shape[-1], 0, kdn.KDN_BF16, kdn.KDN_F32, segments)
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.kdn_scan_kalman_full_noalloc(ctypes.byref(d), p(x["q"]), p(x["k"]), p(x["v"]), p(x["a"]), p(x["r"]),
                                          None, ctypes.c_float(x["qn"]), p(S), p(P), p(o), p(m), stream)


@pytest.mark.gpu
@pytest.mark.parametrize("d", [64, 128])
def test_noalloc_matches_allocating_entry_point_on_two_calls(d):
    w = WORKLOADS["kalman_full_d128"].with_(dk=d, dv=d)
    B, H, T = 1, 3, 200
    S_ref = torch.zeros(B, H, d, d, device="cuda")
    P_ref = torch.eye(d, device="cuda").repeat(B, H, 1, 1)
    S_new, P_new = S_ref.clone(), P_ref.clone()
    for call in range(2):
        x = make_scan_inputs(w, seed=40 + call, device="cuda", B=B, H=H, L=T)
        o_ref, m_ref, _, _ = kdn.scan_kalman_full(x["q"], x["k"], x["v"], x["r"], a=x["a"], qn=x["qn"], S=S_ref,
                                                  P=P_ref)
        o_new = torch.empty(B, H, T, d, device="cuda")
        m_new = torch.empty(B, H, T, device="cuda")
        assert _noalloc_c_abi(x, S_new, P_new, o_new, m_new) == kdn.KDN_OK, kdn.lib().kdn_last_error()
        torch.cuda.synchronize()
        assert kdn.read_device_status(None) == kdn.KDN_OK
        for got, ref in ((o_new, o_ref), (m_new, m_ref), (S_new, S_ref), (P_new, P_ref)):
            assert torch.isfinite(got).all()
            assert _err(got, ref) <= TOL


@pytest.mark.gpu
def test_first_call_with_no_tokens_sets_up_the_array_and_changes_nothing():
    """Callers that reserve device memory at start-up make one call with L = 0 first: it loads the
    array (its first lookup on the device), enqueues only the status-word clear, and leaves S, P alone."""
    B, H, d = 1, 2, 64
    S = torch.randn(B, H, d, d, device="cuda")
    P = torch.eye(d, device="cuda").repeat(B, H, 1, 1) * 2.0
    S0, P0 = S.clone(), P.clone()
    x = {"q": torch.empty(B, H, 0, d, dtype=torch.bfloat16, device="cuda")}
    x["k"], x["v"] = x["q"].clone(), x["q"].clone()
    x["a"] = x["r"] = torch.empty(B, H, 0, device="cuda")
    x["qn"] = 0.0
    o = torch.empty(B, H, 0, d, device="cuda")
    m = torch.empty(B, H, 0, device="cuda")
    assert _noalloc_c_abi(x, S, P, o, m) == kdn.KDN_OK, kdn.lib().kdn_last_error()
    assert kdn.read_device_status(None) == kdn.KDN_OK
    assert torch.equal(S, S0) and torch.equal(P, P0)


@pytest.mark.gpu
def test_at_the_exact_limit_and_one_token_past_it():
    """B*H*L*d_k = 4,194,304 fills the static array exactly and runs; one more token is refused."""
    w = WORKLOADS["kalman_full_d128"]
    B, H, T, d = 1, 4, 8192, 128
    assert B * H * T * d == 4_194_304
    x = make_scan_inputs(w, seed=44, device="cuda", B=B, H=H, L=T)
    S_ref = torch.zeros(B, H, d, d, device="cuda")
    P_ref = torch.eye(d, device="cuda").repeat(B, H, 1, 1)
    S_new, P_new = S_ref.clone(), P_ref.clone()
    o_ref, m_ref, _, _ = kdn.scan_kalman_full(x["q"], x["k"], x["v"], x["r"], a=x["a"], qn=x["qn"], S=S_ref, P=P_ref,
                                              segments=1)
    o_new = torch.empty(B, H, T, d, device="cuda")
    m_new = torch.empty(B, H, T, device="cuda")
    assert _noalloc_c_abi(x, S_new, P_new, o_new, m_new) == kdn.KDN_OK, kdn.lib().kdn_last_error()
    assert kdn.read_device_status(None) == kdn.KDN_OK
    for got, ref in ((o_new, o_ref), (m_new, m_ref), (S_new, S_ref), (P_new, P_ref)):
        assert _err(got, ref) <= TOL
    x1 = make_scan_inputs(w, seed=45, device="cuda", B=B, H=H, L=T + 1)
    o1 = torch.empty(B, H, T + 1, d, device="cuda")
    m1 = torch.empty(B, H, T + 1, device="cuda")
    assert _noalloc_c_abi(x1, S_new, P_new, o1, m1) == kdn.KDN_ERR_UNSUPPORTED
    assert b"needs" in kdn.lib().kdn_last_error()


@pytest.mark.gpu
def test_explicit_segments_that_outgrow_the_array_are_refused_with_their_need():
    w = WORKLOADS["kalman_full_d128"]
    B, H, T, d = 8, 8, 256, 128  # gains 8 MiB fit; two segments add 24 MiB of segment states
    x = make_scan_inputs(w, seed=46, device="cuda", B=B, H=H, L=T)
    S = torch.zeros(B, H, d, d, device="cuda")
    P = torch.eye(d, device="cuda").repeat(B, H, 1, 1)
    o = torch.empty(B, H, T, d, device="cuda")
    m = torch.empty(B, H, T, device="cuda")
    assert _noalloc_c_abi(x, S, P, o, m, segments=2) == kdn.KDN_ERR_UNSUPPORTED
    assert b"2 segments" in kdn.lib().kdn_last_error()


def test_noalloc_rejects_sizes_beyond_its_static_scratch():
    build.build()
    L = kdn.lib()
    d = kdn.Dims(8, 16, 8192, 128, 128, 0, kdn.KDN_BF16, kdn.KDN_F32)  # 134M gains: far beyond 16 MiB
    st = L.kdn_scan_kalman_full_noalloc(ctypes.byref(d), *([None] * 6), ctypes.c_float(0.0), *([None] * 4), None)
    assert st == kdn.KDN_ERR_UNSUPPORTED
    assert b"static array" in L.kdn_last_error()
    assert b"needs" in L.kdn_last_error()


def test_noalloc_refuses_an_explicit_segment_request_it_cannot_serve():
    """Without a GPU driver the chunked path is unavailable, so an explicit split is refused before any
    pointer is looked at; on a GPU the size check words the refusal from the segments' need (above)."""
    build.build()
    L = kdn.lib()
    d = kdn.Dims(1, 1, 256, 128, 128, 0, kdn.KDN_BF16, kdn.KDN_F32, 2)
    st = L.kdn_scan_kalman_full_noalloc(ctypes.byref(d), *([None] * 6), ctypes.c_float(0.0), *([None] * 4), None)
    if not torch.cuda.is_available():
        assert st == kdn.KDN_ERR_UNSUPPORTED
        assert b"segments" in L.kdn_last_error()
    else:
        assert st != kdn.KDN_OK  # NULL pointers: refused either way
