"""Seeded synthetic inputs shaped like the language-model layers the pages train.

This module holds no arithmetic of the method itself: it only draws inputs.
Both the CUDA path (through the binding) and the float64 oracle are fed from
here, so it imports nothing from either.

Recipe (every array is drawn from one ``torch.Generator`` seeded with ``seed``,
in this order): q, k, v, x_beta, x_a, x_r, each standard normal in float32.
q and k are L2-normalised per token in float32 (unit keys on the state path:
A Hippocampus for Linear Attention, sections 3.4-3.5), then rounded to the
input dtype (bf16 or fp32).  v is rounded to the input dtype as drawn.

    beta_t = sigmoid(x_beta)
    a_t    = exp(-softplus(x_a - shift))      shift = 2, or 3 for the full-Kalman layer
    r_t    = softplus(x_r) + 0.1

The scalars stay float32.  Small cases are drawn on the CPU; layer-scale cases
may be drawn directly on the GPU with the same recipe (a different stream of
numbers, equally seeded), and the oracle then reads back the heads it checks.
"""

from __future__ import annotations

from dataclasses import dataclass, field, replace

import torch

__all__ = ["Workload", "WORKLOADS", "make_scan_inputs", "make_decode_inputs"]


@dataclass(frozen=True)
class Workload:
    name: str
    variant: str  # "delta" | "kalman_full" | "kalman_diag" | "kalman_iso"
    B: int
    H: int
    L: int
    dk: int
    dv: int
    dtype: str = "bf16"  # input dtype: "bf16" | "f32"
    a_shift: float | None = 2.0  # None => a_t = 1 (ungated)
    qn: float = 0.0  # process-noise scalar, Q_t = qn * I
    r_const: float | None = None  # None => r_t = softplus(N) + 0.1
    chunk: int = 64
    steps: int = 1  # decode steps (decode workloads only)
    note: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def tokens(self) -> int:
        return self.B * self.H * self.L

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five shapes fixed for this method, plus the delta rule at the diagonal
# layer's shape (the only way to measure the delta scan at d=128, L >= 4096).
WORKLOADS = {
    # tiny oracle check, fp32; the delta run is the plain (ungated) delta rule
    "tiny_delta": Workload("tiny_delta", "delta", 1, 1, 256, 16, 16, "f32", a_shift=None),
    # a=1, Q=0, r=1, P0=I: the Kalman state must equal the ridge closed form
    "tiny_kalman": Workload("tiny_kalman", "kalman_full", 1, 1, 256, 16, 16, "f32", a_shift=None, r_const=1.0),
    "gdn_d64": Workload("gdn_d64", "delta", 4, 8, 2048, 64, 64, "bf16", a_shift=2.0),
    "kalman_full_d128": Workload("kalman_full_d128", "kalman_full", 2, 8, 4096, 128, 128, "bf16", a_shift=3.0, qn=1e-3),
    "kalman_diag_d128": Workload("kalman_diag_d128", "kalman_diag", 8, 16, 8192, 128, 128, "bf16", a_shift=2.0, qn=1e-3),
    "gdn_d128": Workload("gdn_d128", "delta", 8, 16, 8192, 128, 128, "bf16", a_shift=2.0),
    # isotropic Kalman (one uncertainty scalar per head) at the diagonal layer's shape and distributions
    "kalman_iso_d128": Workload("kalman_iso_d128", "kalman_iso", 8, 16, 8192, 128, 128, "bf16", a_shift=2.0, qn=1e-3),
    # decode: batch 256 x 32 heads, one token per call, 1024 calls
    "decode_delta": Workload("decode_delta", "delta", 256, 32, 1, 128, 128, "bf16", a_shift=2.0, steps=1024),
    "decode_diag": Workload("decode_diag", "kalman_diag", 256, 32, 1, 128, 128, "bf16", a_shift=2.0, qn=1e-3, steps=1024),
}


def _dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def _draw(shapes_and_kinds, seed: int, device):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return [torch.randn(s, generator=g, device=device, dtype=torch.float32) for s in shapes_and_kinds]


def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)


def make_scan_inputs(w: Workload, seed: int = 0, device="cpu", B: int | None = None, H: int | None = None,
                     L: int | None = None) -> dict:
    """Inputs for one scan over workload ``w`` (optionally with B, H or L overridden).

    Returns q, k [B,H,L,dk] and v [B,H,L,dv] in the workload dtype, and float32
    beta, a (or None), r [B,H,L], plus the scalar qn.  The initial state is
    S0 = 0, P0 = I (full), p0 = 1 (diagonal) or c0 = 1 (isotropic); the caller allocates it.
    """
    B = w.B if B is None else B
    H = w.H if H is None else H
    L = w.L if L is None else L
    tok = (B, H, L)
    q, k, v, xb, xa, xr = _draw([(*tok, w.dk), (*tok, w.dk), (*tok, w.dv), tok, tok, tok], seed, device)
    dt = _dtype(w.dtype)
    out = {
        "q": _unit(q).to(dt),
        "k": _unit(k).to(dt),
        "v": v.to(dt),
        "beta": torch.sigmoid(xb),
        "a": None if w.a_shift is None else torch.exp(-torch.nn.functional.softplus(xa - w.a_shift)),
        "r": torch.full(tok, float(w.r_const), device=device) if w.r_const is not None
        else torch.nn.functional.softplus(xr) + 0.1,
        "qn": float(w.qn),
    }
    return out


def make_decode_inputs(w: Workload, steps: int | None = None, seed: int = 0, device="cpu",
                       B: int | None = None, H: int | None = None) -> dict:
    """Per-step decode inputs: q, k [steps,B,H,dk], v [steps,B,H,dv], scalars [steps,B,H]."""
    steps = w.steps if steps is None else steps
    B = w.B if B is None else B
    H = w.H if H is None else H
    tok = (steps, B, H)
    q, k, v, xb, xa, xr = _draw([(*tok, w.dk), (*tok, w.dk), (*tok, w.dv), tok, tok, tok], seed, device)
    dt = _dtype(w.dtype)
    return {
        "q": _unit(q).to(dt),
        "k": _unit(k).to(dt),
        "v": v.to(dt),
        "beta": torch.sigmoid(xb),
        "a": None if w.a_shift is None else torch.exp(-torch.nn.functional.softplus(xa - w.a_shift)),
        "r": torch.nn.functional.softplus(xr) + 0.1,
        "qn": float(w.qn),
    }
