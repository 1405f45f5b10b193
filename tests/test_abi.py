"""The C-ABI library builds, loads and exports every entry point include/kdn.h
declares; host-side validation answers without touching a GPU."""

import ctypes

import pytest

from delta_rule_recurrent_scan_b200 import build, kdn


@pytest.fixture(scope="module")
def L():
    build.build()
    return kdn.lib()


def test_every_declared_symbol_is_exported(L):
    names = kdn.exported_names()
    assert {"kdn_scan_delta", "kdn_scan_kalman_full", "kdn_scan_kalman_diag", "kdn_scan_kalman_iso", "kdn_decode_step",
            "kdn_workspace_bytes", "kdn_read_device_status", "kdn_status_string", "kdn_last_error",
            "kdn_api_version", "kdn_scan_kalman_full_noalloc", "kdn_selftest_wait_timeout"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_version_and_status_strings(L):
    assert L.kdn_api_version() == 2
    for code, name in enumerate(["KDN_OK", "KDN_ERR_INVALID_ARG", "KDN_ERR_UNSUPPORTED", "KDN_ERR_CUDA",
                                 "KDN_ERR_NUMERIC", "KDN_ERR_TIMEOUT"]):
        assert L.kdn_status_string(code).decode() == name


def test_workspace_bytes(L):
    d = kdn.Dims(2, 3, 100, 64, 64, 0, kdn.KDN_BF16, kdn.KDN_BF16)
    for v in (0, 1, 2, 3):
        n = L.kdn_workspace_bytes(v, ctypes.byref(d))
        assert n >= 256 and n % 256 == 0
    # the isotropic scan keeps one fp32 beta per token after the status word
    assert L.kdn_workspace_bytes(3, ctypes.byref(d)) >= 256 + 2 * 3 * 100 * 4
    bad = kdn.Dims(2, 3, 100, 48, 64, 0, kdn.KDN_BF16, kdn.KDN_BF16)
    assert L.kdn_workspace_bytes(0, ctypes.byref(bad)) == 0
    assert L.kdn_workspace_bytes(0, None) == 0


def _delta(L, dims, S=None, ws=None, ws_bytes=0):
    return L.kdn_scan_delta(ctypes.byref(dims) if dims is not None else None, None, None, None, None, None, S, None,
                            None, ws, ws_bytes, None)


def test_host_validation_without_gpu(L):
    # null dims, bad sizes and bad dtypes are rejected before any CUDA call
    assert _delta(L, None) == kdn.KDN_ERR_INVALID_ARG
    assert b"dims" in L.kdn_last_error()
    assert _delta(L, kdn.Dims(0, 1, 4, 64, 64, 0, 1, 1)) == kdn.KDN_ERR_INVALID_ARG
    assert _delta(L, kdn.Dims(1, 1, -1, 64, 64, 0, 1, 1)) == kdn.KDN_ERR_INVALID_ARG
    assert _delta(L, kdn.Dims(1, 1, 4, 96, 64, 0, 1, 1)) == kdn.KDN_ERR_UNSUPPORTED
    assert _delta(L, kdn.Dims(1, 1, 4, 64, 64, 48, 1, 1)) == kdn.KDN_ERR_UNSUPPORTED
    assert _delta(L, kdn.Dims(1, 1, 4, 64, 64, 0, 7, 1)) == kdn.KDN_ERR_INVALID_ARG
    # a NULL or misaligned state pointer is caught before its memory type is asked
    assert _delta(L, kdn.Dims(1, 1, 4, 64, 64, 0, 1, 1)) == kdn.KDN_ERR_INVALID_ARG
    assert b"S" in L.kdn_last_error()
    assert _delta(L, kdn.Dims(1, 1, 4, 64, 64, 0, 1, 1), S=ctypes.c_void_p(0x1004)) == kdn.KDN_ERR_INVALID_ARG
    assert b"aligned" in L.kdn_last_error()
    assert L.kdn_decode_step(5, 1, 1, 64, 64, 1, 1, *([None] * 6), 0.0, *([None] * 5)) == kdn.KDN_ERR_UNSUPPORTED
    out = ctypes.c_int(0)
    assert L.kdn_read_device_status(ctypes.c_void_p(0x1000), None, None) == kdn.KDN_ERR_INVALID_ARG
    assert L.kdn_read_device_status(ctypes.c_void_p(0x1004), ctypes.byref(out), None) == kdn.KDN_ERR_INVALID_ARG
    # the failure-path self-test checks its wait limit before it looks at a device
    for bad in (0, -1, 3_000_000_000):
        assert L.kdn_selftest_wait_timeout(None, bad, None) == kdn.KDN_ERR_INVALID_ARG
        assert b"wait_cycles" in L.kdn_last_error()


def test_plan_counts_the_isotropic_prologue(L):
    """The isotropic scan is the delta scan plus a beta prologue, except where the d = 128 chunk kernel
    runs the uncertainty scan itself (which needs a GPU driver to be chosen)."""
    for dims in (kdn.Dims(2, 3, 100, 128, 128, 0, kdn.KDN_BF16, kdn.KDN_F32),
                 kdn.Dims(2, 3, 100, 16, 16, 0, kdn.KDN_F32, kdn.KDN_F32)):
        n_delta, n_iso = ctypes.c_int(-1), ctypes.c_int(-1)
        name = ctypes.c_char_p()
        assert L.kdn_plan(0, ctypes.byref(dims), ctypes.byref(n_delta), ctypes.byref(name), None) == kdn.KDN_OK
        assert L.kdn_plan(3, ctypes.byref(dims), ctypes.byref(n_iso), None, None) == kdn.KDN_OK
        fused = name.value == b"chunk_scan_ws_kernel"
        assert n_iso.value == n_delta.value + (0 if fused else 1)
    assert L.kdn_plan(4, ctypes.byref(kdn.Dims(1, 1, 4, 64, 64, 0, 1, 1)), None, None, None) == kdn.KDN_ERR_INVALID_ARG


def test_segment_requests_on_the_host(L):
    """Segment counts are checked before anything is enqueued: a negative count is invalid, and an explicit
    split needs the chunked path (bf16 inputs, d_k = d_v in {64, 128}; here fp32 at d = 16)."""
    for variant in range(4):
        d = kdn.Dims(1, 1, 64, 16, 16, 0, kdn.KDN_F32, kdn.KDN_F32, -1)
        assert L.kdn_workspace_bytes(variant, ctypes.byref(d)) == 0
        assert L.kdn_plan(variant, ctypes.byref(d), None, None, None) == kdn.KDN_ERR_INVALID_ARG
        d = kdn.Dims(1, 1, 64, 16, 16, 0, kdn.KDN_F32, kdn.KDN_F32, 2)
        assert L.kdn_plan(variant, ctypes.byref(d), None, None, None) == kdn.KDN_ERR_UNSUPPORTED
        assert b"chunked" in L.kdn_last_error()
        auto = kdn.Dims(1, 1, 64, 16, 16, 0, kdn.KDN_F32, kdn.KDN_F32, 0)
        serial = kdn.Dims(1, 1, 64, 16, 16, 0, kdn.KDN_F32, kdn.KDN_F32, 1)
        assert L.kdn_workspace_bytes(variant, ctypes.byref(auto)) == L.kdn_workspace_bytes(variant, ctypes.byref(serial))
    d = kdn.Dims(1, 1, 64, 16, 16, 0, kdn.KDN_F32, kdn.KDN_F32, -1)
    assert _delta(L, d) == kdn.KDN_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors():
    torch = pytest.importorskip("torch")
    q = torch.zeros(1, 1, 4, 16)
    with pytest.raises(ValueError, match="CUDA"):
        kdn.scan_delta(q, q, q, torch.zeros(1, 1, 4))


def test_backward_host_validation(L):
    d = kdn.Dims(2, 3, 100, 64, 32, 0, kdn.KDN_BF16, kdn.KDN_F32)
    n = L.kdn_backward_workspace_bytes(0, ctypes.byref(d))
    # status word + working state + a state per 32-token chunk + one norm per token
    assert n >= 256 + 6 * 64 * 32 * 4 * (1 + 4) + 6 * 100 * 4
    # full Kalman: plus the gains and dG, P at every 32-token block start (4 blocks) and one block's P per token
    assert L.kdn_backward_workspace_bytes(2, ctypes.byref(d)) >= n + 2 * 6 * 100 * 64 * 4 + 6 * (4 + 32) * 64 * 64 * 4
    # isotropic: the delta backward's part plus beta, the uncertainty before every token, ||k||^2 and dbeta
    assert L.kdn_backward_workspace_bytes(3, ctypes.byref(d)) >= n + 4 * 6 * 100 * 4
    # diagonal: plus the gains, the variances before every token and dG
    assert L.kdn_backward_workspace_bytes(1, ctypes.byref(d)) >= n + 3 * 6 * 100 * 64 * 4
    assert L.kdn_scan_delta_backward(None, *([None] * 15), None, 0, None) == kdn.KDN_ERR_INVALID_ARG
    # every output pointer is checked before anything is enqueued
    assert L.kdn_scan_delta_backward(ctypes.byref(d), *([None] * 15), None, 0, None) == kdn.KDN_ERR_INVALID_ARG
    assert b"dS0" in L.kdn_last_error()


def test_iso_backward_host_validation(L):
    d = kdn.Dims(1, 2, 50, 32, 32, 0, kdn.KDN_BF16, kdn.KDN_F32)
    args = [None] * 6 + [0.0] + [None] * 14 + [None, 0, None]
    assert L.kdn_scan_kalman_iso_backward(None, *args) == kdn.KDN_ERR_INVALID_ARG
    # every required pointer is checked before anything is enqueued
    assert L.kdn_scan_kalman_iso_backward(ctypes.byref(d), *args) == kdn.KDN_ERR_INVALID_ARG
    assert b"dS0" in L.kdn_last_error()


def test_hola_workspace_covers_every_block_on_the_tensor_core_path(L):
    tc = kdn.Dims(2, 3, 300, 128, 128, 64, kdn.KDN_BF16, kdn.KDN_F32)
    other = kdn.Dims(2, 3, 300, 64, 64, 64, kdn.KDN_BF16, kdn.KDN_F32)
    assert L.kdn_hola_workspace_bytes(ctypes.byref(tc)) >= 256 + 6 * 5 * 64 * 4
    assert L.kdn_hola_workspace_bytes(ctypes.byref(other)) == 256
    assert L.kdn_hola_workspace_bytes(None) == 0


def test_full_backward_host_validation(L):
    d = kdn.Dims(1, 2, 50, 32, 32, 0, kdn.KDN_BF16, kdn.KDN_F32)
    args = [None] * 6 + [0.0] + [None] * 14 + [None, 0, None]
    assert L.kdn_scan_kalman_full_backward(None, *args) == kdn.KDN_ERR_INVALID_ARG
    assert L.kdn_scan_kalman_full_backward(ctypes.byref(d), *args) == kdn.KDN_ERR_INVALID_ARG
    assert b"dS0" in L.kdn_last_error()
    bad = kdn.Dims(1, 2, 50, 48, 32, 0, kdn.KDN_BF16, kdn.KDN_F32)  # d_k outside 16, 32, 64, 128
    assert L.kdn_backward_workspace_bytes(2, ctypes.byref(bad)) == 0


def test_diag_backward_host_validation(L):
    d = kdn.Dims(1, 2, 50, 32, 32, 0, kdn.KDN_BF16, kdn.KDN_F32)
    args = [None] * 6 + [0.0] + [None] * 14 + [None, 0, None]
    assert L.kdn_scan_kalman_diag_backward(None, *args) == kdn.KDN_ERR_INVALID_ARG
    assert L.kdn_scan_kalman_diag_backward(ctypes.byref(d), *args) == kdn.KDN_ERR_INVALID_ARG
    assert b"dS0" in L.kdn_last_error()
