"""Thin ctypes binding over libkdn.so (the C ABI declared in include/kdn.h).

Argument marshalling only: it checks torch tensors (device, dtype,
contiguity), allocates outputs and default initial states, and passes raw
pointers plus the current CUDA stream to the library.  The read-out o defaults
to fp32: rounding it to bf16 alone costs up to 2^-8 of its magnitude, more than
the 3e-3 the scan is held to; pass out_dtype=torch.bfloat16 to halve its bytes.  Every step of the scan
runs in the library's kernels.  There is no fallback: if the library is
missing or the tensors are not on a CUDA device, the call raises.

Every scan takes ``segments`` (kdn_dims.segments): 0 lets the library cut each
head's sequence into several segments scanned by separate CTAs when there are
too few heads to fill the GPU, 1 forces one serial pass per head, P >= 2 asks
for P segments (P must divide L).  Results agree up to rounding.
"""

from __future__ import annotations

import ctypes
import os
import re

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB_PATH = os.path.join(PKG, "lib", "libkdn.so")
HEADER = os.path.join(ROOT, "include", "kdn.h")

KDN_OK, KDN_ERR_INVALID_ARG, KDN_ERR_UNSUPPORTED, KDN_ERR_CUDA, KDN_ERR_NUMERIC, KDN_ERR_TIMEOUT = range(6)
KDN_F32, KDN_BF16 = 0, 1
VARIANTS = {"delta": 0, "kalman_diag": 1, "kalman_full": 2, "kalman_iso": 3}
_DTYPES = {torch.float32: KDN_F32, torch.bfloat16: KDN_BF16}


class KdnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} (status {status})")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("L", ctypes.c_int), ("dk", ctypes.c_int),
                ("dv", ctypes.c_int), ("chunk", ctypes.c_int), ("in_dtype", ctypes.c_int),
                ("out_dtype", ctypes.c_int), ("segments", ctypes.c_int)]


_lib = None


def exported_names() -> list[str]:
    """The entry points include/kdn.h declares."""
    with open(HEADER) as f:
        return re.findall(r"^KDN_EXPORT\s+[\w\s\*]+?\b(kdn_\w+)\s*\(", f.read(), flags=re.M)


def lib() -> ctypes.CDLL:
    """Open libkdn.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise FileNotFoundError(f"{LIB_PATH} is missing: build it with python -m delta_rule_recurrent_scan_b200.build")
    L = ctypes.CDLL(LIB_PATH)
    vp, sz, i, f = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
    dims = ctypes.POINTER(Dims)
    L.kdn_scan_delta.argtypes = [dims, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.kdn_scan_kalman_full.argtypes = [dims, vp, vp, vp, vp, vp, vp, f, vp, vp, vp, vp, vp, sz, vp]
    L.kdn_scan_kalman_diag.argtypes = [dims, vp, vp, vp, vp, vp, vp, f, vp, vp, vp, vp, vp, sz, vp]
    L.kdn_scan_kalman_iso.argtypes = [dims, vp, vp, vp, vp, vp, vp, f, vp, vp, vp, vp, vp, sz, vp]
    L.kdn_hola_cache_read.argtypes = [dims, vp, vp, vp, vp, vp, vp, vp, i, vp, vp, vp, sz, vp]
    L.kdn_decode_step.argtypes = [i, i, i, i, i, i, i, vp, vp, vp, vp, vp, vp, f, vp, vp, vp, vp, vp]
    L.kdn_scan_kalman_full_noalloc.argtypes = [dims, vp, vp, vp, vp, vp, vp, f, vp, vp, vp, vp, vp]
    L.kdn_scan_kalman_full_noalloc.restype = ctypes.c_int
    L.kdn_workspace_bytes.argtypes = [i, dims]
    L.kdn_workspace_bytes.restype = sz
    L.kdn_read_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int), vp]
    L.kdn_scan_delta_backward.argtypes = [dims] + [vp] * 16 + [sz, vp]
    L.kdn_scan_delta_backward.restype = ctypes.c_int
    L.kdn_hola_workspace_bytes.argtypes = [dims]
    L.kdn_hola_workspace_bytes.restype = sz
    L.kdn_scan_kalman_iso_backward.argtypes = [dims, vp, vp, vp, vp, vp, vp, f] + [vp] * 14 + [vp, sz, vp]
    L.kdn_scan_kalman_iso_backward.restype = ctypes.c_int
    L.kdn_scan_kalman_diag_backward.argtypes = [dims, vp, vp, vp, vp, vp, vp, f] + [vp] * 14 + [vp, sz, vp]
    L.kdn_scan_kalman_diag_backward.restype = ctypes.c_int
    L.kdn_scan_kalman_full_backward.argtypes = [dims, vp, vp, vp, vp, vp, vp, f] + [vp] * 14 + [vp, sz, vp]
    L.kdn_scan_kalman_full_backward.restype = ctypes.c_int
    L.kdn_backward_workspace_bytes.argtypes = [i, dims]
    L.kdn_backward_workspace_bytes.restype = sz
    L.kdn_selftest_wait_timeout.argtypes = [vp, ctypes.c_longlong, vp]
    L.kdn_selftest_wait_timeout.restype = ctypes.c_int
    L.kdn_status_string.argtypes = [i]
    L.kdn_status_string.restype = ctypes.c_char_p
    L.kdn_last_error.argtypes = []
    L.kdn_last_error.restype = ctypes.c_char_p
    L.kdn_api_version.restype = ctypes.c_int
    L.kdn_plan.argtypes = [i, dims, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_char_p),
                           ctypes.POINTER(ctypes.c_char_p)]
    L.kdn_plan.restype = ctypes.c_int
    for name in ("kdn_scan_delta", "kdn_scan_kalman_full", "kdn_scan_kalman_diag", "kdn_decode_step",
                 "kdn_read_device_status"):
        getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def _check(status: int, what: str):
    if status != KDN_OK:
        msg = lib().kdn_last_error().decode()
        raise KdnError(status, f"{what}: {lib().kdn_status_string(status).decode()}: {msg}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, name: str, shape, dtype=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device})")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def workspace_bytes(variant: str, B: int, H: int, L: int, dk: int, dv: int, chunk: int = 0,
                    in_dtype=torch.bfloat16, out_dtype=None, segments: int = 0) -> int:
    d = Dims(B, H, L, dk, dv, chunk, _DTYPES[in_dtype], _DTYPES[out_dtype or torch.float32], segments)
    return int(lib().kdn_workspace_bytes(VARIANTS[variant], ctypes.byref(d)))


def plan(variant: str, B: int, H: int, L: int, dk: int, dv: int, chunk: int = 0, in_dtype=torch.bfloat16,
         out_dtype=None, segments: int = 0) -> dict:
    """The library's own account of the kernels a scan with these sizes runs."""
    d = Dims(B, H, L, dk, dv, chunk, _DTYPES[in_dtype], _DTYPES[out_dtype or torch.float32], segments)
    n, name, arith = ctypes.c_int(0), ctypes.c_char_p(), ctypes.c_char_p()
    _check(lib().kdn_plan(VARIANTS[variant], ctypes.byref(d), ctypes.byref(n), ctypes.byref(name),
                          ctypes.byref(arith)), "kdn_plan")
    return {"launches": n.value, "kernel": name.value.decode(), "arith": arith.value.decode()}


def _scan_common(q, k, v, o, m, S, chunk, out_dtype, segments=0):
    if q.dim() != 4:
        raise ValueError("q must be [B, H, L, d_k]")
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    if q.dtype not in _DTYPES:
        raise ValueError(f"unsupported input dtype {q.dtype}")
    _need(q, "q", (B, H, L, dk), q.dtype)
    _need(k, "k", (B, H, L, dk), q.dtype, dev)
    _need(v, "v", (B, H, L, dv), q.dtype, dev)
    out_dtype = out_dtype or torch.float32
    if o is None:
        o = torch.empty(B, H, L, dv, dtype=out_dtype, device=dev)
    _need(o, "o", (B, H, L, dv), out_dtype, dev)
    if m is None:
        m = torch.empty(B, H, L, dtype=torch.float32, device=dev)
    _need(m, "m", (B, H, L), torch.float32, dev)
    if S is None:
        S = torch.zeros(B, H, dk, dv, dtype=torch.float32, device=dev)
    _need(S, "S", (B, H, dk, dv), torch.float32, dev)
    dims = Dims(B, H, L, dk, dv, chunk, _DTYPES[q.dtype], _DTYPES[out_dtype], segments)
    return dims, o, m, S


def _workspace(variant, dims, workspace, dev):
    need = int(lib().kdn_workspace_bytes(VARIANTS[variant], ctypes.byref(dims)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    if workspace.device.type != "cuda" or workspace.dtype != torch.uint8 or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous uint8 CUDA tensor")
    return workspace


def scan_delta(q, k, v, beta, a=None, S=None, o=None, m=None, workspace=None, chunk=0, out_dtype=None, segments=0,
               stream=None):
    """Gated delta rule scan.  Returns (o, m, S); S is updated in place when given."""
    dims, o, m, S = _scan_common(q, k, v, o, m, S, chunk, out_dtype, segments)
    tok = tuple(q.shape[:3])
    _need(beta, "beta", tok, torch.float32, q.device)
    if a is not None:
        _need(a, "a", tok, torch.float32, q.device)
    workspace = _workspace("delta", dims, workspace, q.device)
    st = lib().kdn_scan_delta(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(a), _ptr(S), _ptr(o),
                              _ptr(m), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "kdn_scan_delta")
    return o, m, S


def scan_delta_backward(q, k, v, beta, dO, a=None, S0=None, dm=None, dS_L=None, workspace=None, stream=None,
                        want_da=True):
    """Gradients of the gated delta rule scan for upstream dO (and dm, dS_L).  Returns a dict with dq, dk,
    dv, dbeta, da (None if not wanted) and dS0, all fp32."""
    if q.dim() != 4:
        raise ValueError("q must be [B, H, L, d_k]")
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    if q.dtype not in _DTYPES:
        raise ValueError(f"unsupported input dtype {q.dtype}")
    _need(q, "q", (B, H, L, dk), q.dtype)
    _need(k, "k", (B, H, L, dk), q.dtype, dev)
    _need(v, "v", (B, H, L, dv), q.dtype, dev)
    tok = (B, H, L)
    _need(beta, "beta", tok, torch.float32, dev)
    _need(dO, "dO", (B, H, L, dv), torch.float32, dev)
    for name, t, shape in (("a", a, tok), ("dm", dm, tok), ("S0", S0, (B, H, dk, dv)), ("dS_L", dS_L, (B, H, dk, dv))):
        if t is not None:
            _need(t, name, shape, torch.float32, dev)
    out = {"dq": torch.empty(B, H, L, dk, device=dev), "dk": torch.empty(B, H, L, dk, device=dev),
           "dv": torch.empty(B, H, L, dv, device=dev), "dbeta": torch.empty(B, H, L, device=dev),
           "da": torch.empty(B, H, L, device=dev) if want_da else None,
           "dS0": torch.empty(B, H, dk, dv, device=dev)}
    dims = Dims(B, H, L, dk, dv, 0, _DTYPES[q.dtype], KDN_F32, 0)
    need = int(lib().kdn_backward_workspace_bytes(VARIANTS["delta"], ctypes.byref(dims)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    st = lib().kdn_scan_delta_backward(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(a), _ptr(S0),
                                       _ptr(dO), _ptr(dm), _ptr(dS_L), _ptr(out["dq"]), _ptr(out["dk"]),
                                       _ptr(out["dv"]), _ptr(out["dbeta"]), _ptr(out["da"]), _ptr(out["dS0"]),
                                       _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "kdn_scan_delta_backward")
    return out


def scan_kalman_diag_backward(q, k, v, r, dO, a=None, qn=None, S0=None, p0=None, dm=None, dS_L=None, dp_L=None,
                              workspace=None, stream=None, want_da=True):
    """Gradients of the diagonal Kalman scan for upstream dO (and dm, dS_L, dp_L).  Returns a dict with dq, dk,
    dv, dr, da (None if not wanted), dqn (per token), dS0 and dp0, all fp32."""
    return _kalman_backward("kalman_diag", q, k, v, r, dO, a, qn, S0, p0, dm, dS_L, dp_L, workspace, stream, want_da)


def scan_kalman_iso_backward(q, k, v, r, dO, a=None, qn=None, S0=None, c0=None, dm=None, dS_L=None, dc_L=None,
                             workspace=None, stream=None, want_da=True):
    """Gradients of the isotropic Kalman scan for upstream dO (and dm, dS_L, dc_L).  Returns a dict with dq, dk,
    dv, dr, da (None if not wanted), dqn (per token), dS0 and dc0, all fp32."""
    return _kalman_backward("kalman_iso", q, k, v, r, dO, a, qn, S0, c0, dm, dS_L, dc_L, workspace, stream, want_da)


def scan_kalman_full_backward(q, k, v, r, dO, a=None, qn=None, S0=None, P0=None, dm=None, dS_L=None, dP_L=None,
                              workspace=None, stream=None, want_da=True):
    """Gradients of the full-covariance Kalman scan for upstream dO (and dm, dS_L, dP_L).  Returns a dict with dq,
    dk, dv, dr, da (None if not wanted), dqn (per token), dS0 and dP0 (the gradient for a symmetric P0), all fp32."""
    return _kalman_backward("kalman_full", q, k, v, r, dO, a, qn, S0, P0, dm, dS_L, dP_L, workspace, stream, want_da)


def _kalman_backward(variant, q, k, v, r, dO, a, qn, S0, u0, dm, dS_L, du_L, workspace, stream, want_da):
    """The uncertainty-side backward shared by the isotropic (u = c, one per head), diagonal (u = p, one per
    coordinate) and full (u = P, d_k x d_k per head) variants."""
    if q.dim() != 4:
        raise ValueError("q must be [B, H, L, d_k]")
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    if q.dtype not in _DTYPES:
        raise ValueError(f"unsupported input dtype {q.dtype}")
    _need(q, "q", (B, H, L, dk), q.dtype)
    _need(k, "k", (B, H, L, dk), q.dtype, dev)
    _need(v, "v", (B, H, L, dv), q.dtype, dev)
    tok = (B, H, L)
    _need(r, "r", tok, torch.float32, dev)
    _need(dO, "dO", (B, H, L, dv), torch.float32, dev)
    ushape = {"kalman_iso": (B, H), "kalman_diag": (B, H, dk), "kalman_full": (B, H, dk, dk)}[variant]
    uname = {"kalman_iso": "c", "kalman_diag": "p", "kalman_full": "P"}[variant]
    for name, t, shape in (("a", a, tok), ("dm", dm, tok), ("S0", S0, (B, H, dk, dv)), ("dS_L", dS_L, (B, H, dk, dv)),
                           (uname + "0", u0, ushape), ("d" + uname + "_L", du_L, ushape)):
        if t is not None:
            _need(t, name, shape, torch.float32, dev)
    qn_t, qn_s = _qn_args(qn, tok, dev)
    out = {"dq": torch.empty(B, H, L, dk, device=dev), "dk": torch.empty(B, H, L, dk, device=dev),
           "dv": torch.empty(B, H, L, dv, device=dev), "dr": torch.empty(B, H, L, device=dev),
           "da": torch.empty(B, H, L, device=dev) if want_da else None, "dqn": torch.empty(B, H, L, device=dev),
           "dS0": torch.empty(B, H, dk, dv, device=dev), "d" + uname + "0": torch.empty(*ushape, device=dev)}
    dims = Dims(B, H, L, dk, dv, 0, _DTYPES[q.dtype], KDN_F32, 0)
    need = int(lib().kdn_backward_workspace_bytes(VARIANTS[variant], ctypes.byref(dims)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    fn = {"kalman_iso": lib().kdn_scan_kalman_iso_backward, "kalman_diag": lib().kdn_scan_kalman_diag_backward,
          "kalman_full": lib().kdn_scan_kalman_full_backward}[variant]
    st = fn(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(r), _ptr(a), _ptr(qn_t), qn_s, _ptr(S0), _ptr(u0),
            _ptr(dO), _ptr(dm), _ptr(dS_L), _ptr(du_L), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
            _ptr(out["dr"]), _ptr(out["da"]), _ptr(out["dqn"]), _ptr(out["dS0"]), _ptr(out["d" + uname + "0"]),
            _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "kdn_scan_" + variant + "_backward")
    return out


def _qn_args(qn, tok, dev):
    if qn is None:
        return None, 0.0
    if isinstance(qn, (int, float)):
        return None, float(qn)
    _need(qn, "qn", tok, torch.float32, dev)
    return qn, 0.0


def scan_kalman_full(q, k, v, r, a=None, qn=None, S=None, P=None, o=None, m=None, workspace=None, chunk=0,
                     out_dtype=None, segments=0, stream=None):
    """Full-covariance Kalman scan.  Returns (o, m, S, P); S and P are updated in place when given."""
    dims, o, m, S = _scan_common(q, k, v, o, m, S, chunk, out_dtype, segments)
    B, H, L, dk = q.shape
    tok = (B, H, L)
    _need(r, "r", tok, torch.float32, q.device)
    if a is not None:
        _need(a, "a", tok, torch.float32, q.device)
    qn_t, qn_s = _qn_args(qn, tok, q.device)
    if P is None:
        P = torch.eye(dk, dtype=torch.float32, device=q.device).repeat(B, H, 1, 1)
    _need(P, "P", (B, H, dk, dk), torch.float32, q.device)
    workspace = _workspace("kalman_full", dims, workspace, q.device)
    st = lib().kdn_scan_kalman_full(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(r), _ptr(qn_t), qn_s,
                                    _ptr(S), _ptr(P), _ptr(o), _ptr(m), _ptr(workspace), workspace.numel(),
                                    _stream(stream))
    _check(st, "kdn_scan_kalman_full")
    return o, m, S, P


def scan_kalman_full_noalloc(q, k, v, r, a=None, qn=None, S=None, P=None, o=None, m=None, chunk=0,
                             out_dtype=None, segments=0, stream=None):
    """Full-Kalman scan without a workspace, for callers that cannot allocate one: the library uses a static
    device array (B*H*L*d_k <= 4,194,304; overlapping calls race on it).  Returns (o, m, S, P)."""
    dims, o, m, S = _scan_common(q, k, v, o, m, S, chunk, out_dtype, segments)
    B, H, L, dk = q.shape
    tok = (B, H, L)
    _need(r, "r", tok, torch.float32, q.device)
    if a is not None:
        _need(a, "a", tok, torch.float32, q.device)
    qn_t, qn_s = _qn_args(qn, tok, q.device)
    if P is None:
        P = torch.eye(dk, dtype=torch.float32, device=q.device).repeat(B, H, 1, 1)
    _need(P, "P", (B, H, dk, dk), torch.float32, q.device)
    st = lib().kdn_scan_kalman_full_noalloc(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(r),
                                            _ptr(qn_t), qn_s, _ptr(S), _ptr(P), _ptr(o), _ptr(m), _stream(stream))
    _check(st, "kdn_scan_kalman_full_noalloc")
    return o, m, S, P


def scan_kalman_diag(q, k, v, r, a=None, qn=None, S=None, p=None, o=None, m=None, workspace=None, chunk=0,
                     out_dtype=None, segments=0, stream=None):
    """Diagonal-covariance Kalman scan.  Returns (o, m, S, p); S and p are updated in place when given."""
    dims, o, m, S = _scan_common(q, k, v, o, m, S, chunk, out_dtype, segments)
    B, H, L, dk = q.shape
    tok = (B, H, L)
    _need(r, "r", tok, torch.float32, q.device)
    if a is not None:
        _need(a, "a", tok, torch.float32, q.device)
    qn_t, qn_s = _qn_args(qn, tok, q.device)
    if p is None:
        p = torch.ones(B, H, dk, dtype=torch.float32, device=q.device)
    _need(p, "p", (B, H, dk), torch.float32, q.device)
    workspace = _workspace("kalman_diag", dims, workspace, q.device)
    st = lib().kdn_scan_kalman_diag(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(r), _ptr(qn_t), qn_s,
                                    _ptr(S), _ptr(p), _ptr(o), _ptr(m), _ptr(workspace), workspace.numel(),
                                    _stream(stream))
    _check(st, "kdn_scan_kalman_diag")
    return o, m, S, p


def scan_kalman_iso(q, k, v, r, a=None, qn=None, S=None, c=None, o=None, m=None, workspace=None, chunk=0,
                    out_dtype=None, segments=0, stream=None):
    """Isotropic-covariance Kalman scan (one uncertainty scalar per head).  Returns (o, m, S, c); S and c
    are updated in place when given."""
    dims, o, m, S = _scan_common(q, k, v, o, m, S, chunk, out_dtype, segments)
    B, H, L, dk = q.shape
    tok = (B, H, L)
    _need(r, "r", tok, torch.float32, q.device)
    if a is not None:
        _need(a, "a", tok, torch.float32, q.device)
    qn_t, qn_s = _qn_args(qn, tok, q.device)
    if c is None:
        c = torch.ones(B, H, dtype=torch.float32, device=q.device)
    _need(c, "c", (B, H), torch.float32, q.device)
    workspace = _workspace("kalman_iso", dims, workspace, q.device)
    st = lib().kdn_scan_kalman_iso(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(r), _ptr(qn_t), qn_s,
                                   _ptr(S), _ptr(c), _ptr(o), _ptr(m), _ptr(workspace), workspace.numel(),
                                   _stream(stream))
    _check(st, "kdn_scan_kalman_iso")
    return o, m, S, c


def hola_cache_read(q, k, v, m, gamma_q, gamma_k, sink, w=64, block=64, o=None, cache=None, workspace=None,
                    stream=None):
    """Surprise-cache read: q, k [B,H,L,d_k], v [B,H,L,d_v] (bf16 or fp32), m [B,H,L], gamma_q/gamma_k [d_k],
    sink [H].  Returns (o_cache [B,H,L,d_v] fp32, cache [B,H,w] int32 token indices, ascending, -1 empty)."""
    if q.dim() != 4:
        raise ValueError("q must be [B, H, L, d_k]")
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    _need(q, "q", (B, H, L, dk), q.dtype)
    _need(k, "k", (B, H, L, dk), q.dtype, dev)
    _need(v, "v", (B, H, L, dv), q.dtype, dev)
    _need(m, "m", (B, H, L), torch.float32, dev)
    _need(gamma_q, "gamma_q", (dk,), torch.float32, dev)
    _need(gamma_k, "gamma_k", (dk,), torch.float32, dev)
    _need(sink, "sink", (H,), torch.float32, dev)
    if o is None:
        o = torch.empty(B, H, L, dv, dtype=torch.float32, device=dev)
    _need(o, "o", (B, H, L, dv), torch.float32, dev)
    if cache is None:
        cache = torch.empty(B, H, w, dtype=torch.int32, device=dev)
    _need(cache, "cache", (B, H, w), torch.int32, dev)
    dims = Dims(B, H, L, dk, dv, block, _DTYPES[q.dtype], KDN_F32)
    if workspace is None:
        need = int(lib().kdn_hola_workspace_bytes(ctypes.byref(dims)))
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    st = lib().kdn_hola_cache_read(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(m), _ptr(gamma_q),
                                   _ptr(gamma_k), _ptr(sink), int(w), _ptr(o), _ptr(cache), _ptr(workspace),
                                   workspace.numel(), _stream(stream))
    _check(st, "kdn_hola_cache_read")
    return o, cache


def decode_step(variant, q, k, v, S, beta=None, a=None, r=None, qn=0.0, p=None, o=None, m=None, out_dtype=None,
                stream=None):
    """One token per head against a resident state.  q, k [B,H,d_k], v [B,H,d_v]; S (and p: the diagonal
    variances [B,H,d_k], or for "kalman_iso" the uncertainty scalar [B,H]) updated in place.  Returns (o, m)."""
    if q.dim() != 3:
        raise ValueError("q must be [B, H, d_k]")
    B, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    _need(q, "q", (B, H, dk), q.dtype)
    _need(k, "k", (B, H, dk), q.dtype, dev)
    _need(v, "v", (B, H, dv), q.dtype, dev)
    _need(S, "S", (B, H, dk, dv), torch.float32, dev)
    out_dtype = out_dtype or torch.float32
    if o is None:
        o = torch.empty(B, H, dv, dtype=out_dtype, device=dev)
    _need(o, "o", (B, H, dv), out_dtype, dev)
    if m is None:
        m = torch.empty(B, H, dtype=torch.float32, device=dev)
    _need(m, "m", (B, H), torch.float32, dev)
    for name, t in (("beta", beta), ("a", a), ("r", r)):
        if t is not None:
            _need(t, name, (B, H), torch.float32, dev)
    if p is not None:  # diagonal: p [B,H,d_k]; isotropic: the uncertainty scalar c [B,H]
        _need(p, "p", (B, H) if variant == "kalman_iso" else (B, H, dk), torch.float32, dev)
    st = lib().kdn_decode_step(VARIANTS[variant], B, H, dk, dv, _DTYPES[q.dtype], _DTYPES[out_dtype], _ptr(q), _ptr(k),
                               _ptr(v), _ptr(beta), _ptr(a), _ptr(r), float(qn), _ptr(S), _ptr(p), _ptr(o), _ptr(m),
                               _stream(stream))
    _check(st, "kdn_decode_step")
    return o, m


def read_device_status(workspace: torch.Tensor | None, stream=None) -> int:
    """Synchronise the stream and return the device status of a scan's workspace (a KDN_* code).
    ``workspace=None`` reads the status word of the no-alloc full-Kalman scan on the current device."""
    out = ctypes.c_int(-1)
    st = lib().kdn_read_device_status(_ptr(workspace), ctypes.byref(out), _stream(stream))
    _check(st, "kdn_read_device_status")
    return out.value


def selftest_wait_timeout(workspace: torch.Tensor | None, wait_cycles: int = 100_000, stream=None) -> None:
    """Run the bounded-wait failure path once on purpose (a wait on an mbarrier nothing arrives at, with
    nothing in flight): afterwards ``read_device_status(workspace)`` reports KDN_ERR_TIMEOUT."""
    st = lib().kdn_selftest_wait_timeout(_ptr(workspace), int(wait_cycles), _stream(stream))
    _check(st, "kdn_selftest_wait_timeout")
