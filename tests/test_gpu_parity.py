"""GPU parity: the CUDA path, called through the C ABI, against the float64 oracle.

Sizes here span several 64-token chunks and a ragged tail; the layer-scale
workloads run at full size in the launch configuration the benchmark times and
are checked on sampled heads over the whole sequence.  Tolerances (normwise per
head): 1e-4 for fp32 inputs, 3e-3 for bf16 inputs.  The read-out o is fp32 by
default; a bf16 o is held to the same tolerance beyond its own rounding (bf16
keeps 8 significand bits, so rounding alone may cost 2^-8 > 3e-3).
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
from delta_rule_recurrent_scan_b200 import kdn
from delta_rule_recurrent_scan_b200.workloads import WORKLOADS, make_decode_inputs, make_scan_inputs
from parity import TOL, assert_symmetric_pd, compare, initial_state, normwise_err, run_gpu, run_oracle, self_tol

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _to(x, device):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


# ----------------------------------------------------------------------------- tiny fp32 workloads


def test_tiny_delta_fp32():
    w = WORKLOADS["tiny_delta"]
    x = _to(make_scan_inputs(w, seed=0), DEV)
    got = run_gpu("delta", x)
    compare(got, run_oracle("delta", x), TOL["f32"])


def test_tiny_kalman_fp32_matches_oracle_and_ridge():
    w = WORKLOADS["tiny_kalman"]
    x = _to(make_scan_inputs(w, seed=0), DEV)
    got = run_gpu("kalman_full", x)
    compare(got, run_oracle("kalman_full", x), TOL["f32"])
    K = x["k"][0, 0].double().cpu().numpy()
    V = x["v"][0, 0].double().cpu().numpy()
    S_ridge = np.linalg.solve(np.eye(16) + K.T @ K, K.T @ V)
    assert normwise_err(got["S"][0, 0][None, None], S_ridge[None, None]) < TOL["f32"]
    P_ridge = np.linalg.inv(np.eye(16) + K.T @ K)
    assert normwise_err(got["P"][0, 0][None, None], P_ridge[None, None]) < TOL["f32"]


def test_tiny_isotropic_fp32_and_a_long_sequence():
    """The isotropic prologue scans its per-head Moebius maps in tiles of 2048 tokens: a sequence of
    several tiles (with a ragged last one) checks the carry between tiles."""
    w = WORKLOADS["tiny_kalman"].with_(variant="kalman_iso", a_shift=2.0, qn=1e-3, r_const=None)
    x = _to(make_scan_inputs(w, seed=0), DEV)
    compare(run_gpu("kalman_iso", x), run_oracle("kalman_iso", x), TOL["f32"])
    x = make_scan_inputs(w, seed=1, device=DEV, B=1, H=3, L=5000)
    got = run_gpu("kalman_iso", x)
    compare(got, run_oracle("kalman_iso", x), TOL["f32"])


# ----------------------------------------------------------------------------- reduced layer shapes


@pytest.mark.parametrize("name,B,H,L", [
    ("gdn_d64", 2, 2, 300),
    ("gdn_d128", 1, 2, 300),
    ("kalman_diag_d128", 1, 2, 300),
    ("kalman_full_d128", 1, 2, 200),
    ("kalman_iso_d128", 1, 2, 300),
])
def test_layer_shapes_reduced(name, B, H, L):
    w = WORKLOADS[name]
    x = make_scan_inputs(w, seed=1, device=DEV, B=B, H=H, L=L)
    got = run_gpu(w.variant, x)
    compare(got, run_oracle(w.variant, x), TOL["bf16"])


@pytest.mark.parametrize("variant", ["delta", "kalman_diag", "kalman_full", "kalman_iso"])
@pytest.mark.parametrize("dk,dv", [(64, 32), (32, 128), (16, 64), (128, 16)])
def test_unequal_head_dims(variant, dk, dv):
    w = WORKLOADS["gdn_d64"].with_(variant=variant, dk=dk, dv=dv, qn=1e-3)
    x = make_scan_inputs(w, seed=2, device=DEV, B=1, H=2, L=130)
    got = run_gpu(variant, x)
    compare(got, run_oracle(variant, x), TOL["bf16"])


@pytest.mark.parametrize("variant", ["delta", "kalman_diag", "kalman_full", "kalman_iso"])
def test_bf16_output_within_tolerance_beyond_its_rounding(variant):
    w = WORKLOADS["gdn_d128"].with_(variant=variant, qn=1e-3)
    x = make_scan_inputs(w, seed=13, device=DEV, B=1, H=2, L=200)
    got = run_gpu(variant, x, out_dtype=torch.bfloat16)
    assert got["o"].dtype == torch.bfloat16
    compare(got, run_oracle(variant, x), TOL["bf16"])


@pytest.mark.parametrize("variant", ["delta", "kalman_diag", "kalman_full", "kalman_iso"])
def test_fp32_inputs_d64(variant):
    w = WORKLOADS["gdn_d64"].with_(variant=variant, dtype="f32", qn=1e-3)
    x = make_scan_inputs(w, seed=3, device=DEV, B=1, H=2, L=150)
    compare(run_gpu(variant, x), run_oracle(variant, x), TOL["f32"])


@pytest.mark.parametrize("variant", ["delta", "kalman_diag", "kalman_full", "kalman_iso"])
@pytest.mark.parametrize("d", [64, 128])
def test_tensor_core_path_matches_per_token_path(variant, d):
    """chunk=0 takes the chunked tcgen05 kernel for bf16 d in {64, 128}; chunk=32 the per-token kernels."""
    w = WORKLOADS["gdn_d128"].with_(variant=variant, dk=d, dv=d, qn=1e-3)
    plan = kdn.plan(variant, 1, 3, 333, d, d)
    assert plan["arith"] == "bf16-tc", plan
    x = make_scan_inputs(w, seed=14, device=DEV, B=1, H=3, L=333)
    fast = run_gpu(variant, x)
    slow = run_gpu(variant, x, chunk=32)
    for key in fast:
        assert normwise_err(fast[key], slow[key]) < 1e-3, key
    compare(fast, run_oracle(variant, x), TOL["bf16"])


@pytest.mark.parametrize("variant", ["delta", "kalman_diag", "kalman_full", "kalman_iso"])
@pytest.mark.parametrize("d", [64, 128])
def test_results_do_not_depend_on_the_chunk_size(variant, d):
    """Every chunk size the library accepts (0 = its choice, 16, 32, 64) gives the same scan: to the
    rounding of the tensor-core splits between chunkings, and to the oracle's tolerance for each."""
    w = WORKLOADS["gdn_d128"].with_(variant=variant, dk=d, dv=d, qn=1e-3)
    x = make_scan_inputs(w, seed=15, device=DEV, B=1, H=2, L=333)
    ref = run_oracle(variant, x)
    runs = {C: run_gpu(variant, x, chunk=C) for C in (0, 16, 32, 64)}
    for C, got in runs.items():
        compare(got, ref, TOL["bf16"])
        for key in got:
            assert normwise_err(got[key], runs[64][key]) < 1e-3, (C, key)


# ----------------------------------------------------------------------------- edge cases


@pytest.mark.parametrize("variant", ["delta", "kalman_diag", "kalman_full", "kalman_iso"])
def test_empty_sequence_is_a_no_op(variant):
    w = WORKLOADS["gdn_d64"].with_(variant=variant)
    x = make_scan_inputs(w, seed=4, device=DEV, B=2, H=2, L=0)
    S, C = initial_state(variant, 2, 2, 64, 64, DEV)
    S += 0.5
    S0 = S.clone()
    got = run_gpu(variant, x, S=S, C=C)
    torch.cuda.synchronize()
    assert torch.equal(got["S"], S0)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("variant", ["delta", "kalman_diag", "kalman_full", "kalman_iso"])
def test_single_token_and_degenerate_gates(variant, d):
    w = WORKLOADS["gdn_d64"].with_(variant=variant, qn=1e-3, dk=d, dv=d)
    x = make_scan_inputs(w, seed=5, device=DEV, B=2, H=2, L=97)
    x["a"][:, :, ::7] = 0.0   # full resets
    x["a"][:, :, 3::11] = 1.0  # no decay
    x["beta"][:, :, 5::13] = 0.0  # no write
    x["beta"][:, :, 6::13] = 1.0
    compare(run_gpu(variant, x), run_oracle(variant, x), TOL["bf16"])
    x1 = make_scan_inputs(w, seed=6, device=DEV, B=2, H=2, L=1)
    compare(run_gpu(variant, x1), run_oracle(variant, x1), TOL["bf16"])


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("variant", ["kalman_diag", "kalman_full"])
def test_cancelling_single_token_readout(variant, d):
    """One token per head with q nearly orthogonal to k: o_1 = (q . g) v_1 with q . g about 1e-3 of |q| |g|.
    The read-out's q . g must then carry the gain's rounding relative to itself, not to |q| |g| (a single fp16
    rounding of the gains would leave a few per cent here)."""
    w = WORKLOADS["gdn_d64"].with_(variant=variant, qn=1e-3, dk=d, dv=d)
    x = make_scan_inputs(w, seed=9, device=DEV, B=1, H=8, L=1)
    k = x["k"].float()
    u = torch.randn(k.shape, generator=torch.Generator(device="cpu").manual_seed(10)).to(DEV)
    u = u - (u * k).sum(-1, keepdim=True) * k  # orthogonal to k
    q = u / u.norm(dim=-1, keepdim=True) + 1e-3 * k
    x["q"] = q.to(x["q"].dtype)
    qk = (x["q"].float() * k).sum(-1).abs().max().item()
    assert qk < 3e-3, qk  # the bf16 rounding of q keeps q . k small
    compare(run_gpu(variant, x), run_oracle(variant, x), TOL["bf16"])


@pytest.mark.parametrize("variant", ["delta", "kalman_diag", "kalman_full", "kalman_iso"])
def test_split_invariance_and_resume(variant):
    """scan(x_1..L) equals scan(x_1..L1) then scan(x_L1+1..L) with the state passed through."""
    w = WORKLOADS["gdn_d64"].with_(variant=variant, qn=1e-3)
    x = make_scan_inputs(w, seed=7, device=DEV, B=1, H=2, L=200)
    whole = run_gpu(variant, x)
    S, C = initial_state(variant, 1, 2, 64, 64, DEV)
    parts = []
    for lo, hi in ((0, 77), (77, 200)):
        xs = {k: (v[:, :, lo:hi].contiguous() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
        out = run_gpu(variant, xs, S=S, C=C)
        parts.append(out)
    o = torch.cat([p["o"] for p in parts], dim=2)
    # a different chunking rounds differently: the fp16 operands carry 2^-11
    assert normwise_err(o.float(), whole["o"].float()) < self_tol(64)
    assert normwise_err(S, whole["S"]) < self_tol(64)


# ----------------------------------------------------------------------------- full layer-scale workloads


def _sample_heads(B, H, n=2, seed=0):
    g = np.random.default_rng(seed)
    return [(int(g.integers(B)), int(g.integers(H))) for _ in range(n)]


@pytest.mark.parametrize("name", ["gdn_d64", "kalman_full_d128", "kalman_diag_d128", "gdn_d128", "kalman_iso_d128"])
def test_full_size_sampled_heads(name):
    w = WORKLOADS[name]
    x = make_scan_inputs(w, seed=0, device=DEV)
    got = run_gpu(w.variant, x)
    heads = _sample_heads(w.B, w.H)
    ref = run_oracle(w.variant, x, heads=heads)
    compare(got, ref, TOL["bf16"], heads=heads)
    if w.variant == "kalman_full":
        assert_symmetric_pd(got["P"])


# ----------------------------------------------------------------------------- decode


@pytest.mark.parametrize("variant", ["delta", "kalman_diag", "kalman_iso"])
def test_decode_steps_equal_scan_and_oracle(variant):
    name = "decode_delta" if variant == "delta" else "decode_diag"
    w = WORKLOADS[name]
    steps, B, H = 8, 4, 3
    x = make_decode_inputs(w, steps=steps, seed=8, device=DEV, B=B, H=H)
    S, C = initial_state(variant, B, H, w.dk, w.dv, DEV)
    outs, ms = [], []
    for t in range(steps):
        o, m = kdn.decode_step(variant, x["q"][t], x["k"][t], x["v"][t], S, beta=x["beta"][t], a=x["a"][t],
                               r=x["r"][t], qn=x["qn"], p=C)
        outs.append(o)
        ms.append(m)
    # the same tokens as one scan (layout [B, H, L, d])
    xs = {k: (v.movedim(0, 2).contiguous() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    scan = run_gpu(variant, xs)
    o = torch.stack(outs, dim=2)
    assert normwise_err(o.float(), scan["o"].float()) < self_tol(w.dk)  # the scan takes the chunk kernel
    assert normwise_err(S, scan["S"]) < self_tol(w.dk)
    ref = run_oracle(variant, xs)
    compare({"o": o, "m": torch.stack(ms, dim=2), "S": S}, ref, TOL["bf16"])
    if variant == "kalman_diag":
        compare({"p": C}, {"p": ref["p"]}, TOL["bf16"])
    if variant == "kalman_iso":
        compare({"c": C}, {"c": ref["c"]}, TOL["bf16"])


@pytest.mark.parametrize("name", ["decode_delta", "decode_diag"])
def test_decode_full_batch_sampled_heads(name):
    w = WORKLOADS[name]
    variant = w.variant
    steps = 4
    x = make_decode_inputs(w, steps=steps, seed=9, device=DEV)
    S, C = initial_state(variant, w.B, w.H, w.dk, w.dv, DEV)
    S.normal_(0.0, 0.1, generator=torch.Generator(device=DEV).manual_seed(3))
    S0 = S.clone()
    C0 = None if C is None else C.clone()
    for t in range(steps):
        o, m = kdn.decode_step(variant, x["q"][t], x["k"][t], x["v"][t], S, beta=x["beta"][t], a=x["a"][t],
                               r=x["r"][t], qn=x["qn"], p=C)
    heads = _sample_heads(w.B, w.H, n=3, seed=1)
    pick = lambda t: np.stack([t[:, b, h].double().cpu().numpy() for b, h in heads], axis=0)[None]  # noqa: E731
    pick0 = lambda t: np.stack([t[b, h].double().cpu().numpy() for b, h in heads], axis=0)[None]  # noqa: E731
    if variant == "delta":
        ref = oracle.scan_delta(pick(x["q"]), pick(x["k"]), pick(x["v"]), pick(x["beta"]), a=pick(x["a"]),
                                S0=pick0(S0))
    else:
        ref = oracle.scan_kalman_diag(pick(x["q"]), pick(x["k"]), pick(x["v"]), r=pick(x["r"]), a=pick(x["a"]),
                                      qn=x["qn"], S0=pick0(S0), p0=pick0(C0))
    got_S = torch.stack([S[b, h] for b, h in heads])[None]
    assert normwise_err(got_S, ref["S"]) < TOL["bf16"]
    got_o = torch.stack([o[b, h] for b, h in heads])[None]
    assert normwise_err(got_o.float()[:, :, None], ref["o"][:, :, -1:]) < TOL["bf16"]


@pytest.mark.parametrize("name", ["decode_delta", "decode_diag"])
def test_decode_1024_steps_full_batch_sampled_heads(name):
    """The decode workload as specified: 1024 one-token calls over the full batch (256 x 32 heads), each
    step's inputs drawn fresh; three sampled heads are followed by the oracle over all 1024 tokens (o and
    m at every step, S and p at the end), so that error growth over a long decode would show."""
    w = WORKLOADS[name]
    variant, steps = w.variant, w.steps
    assert steps == 1024
    S, C = initial_state(variant, w.B, w.H, w.dk, w.dv, DEV)
    heads = _sample_heads(w.B, w.H, n=3, seed=2)
    bi = torch.tensor([b for b, _ in heads], device=DEV)
    hi = torch.tensor([h for _, h in heads], device=DEV)
    seen = {key: [] for key in ("q", "k", "v", "beta", "a", "r")}
    outs, ms = [], []
    for t in range(steps):
        x = make_decode_inputs(w, steps=1, seed=1000 + t, device=DEV)
        o, m = kdn.decode_step(variant, x["q"][0], x["k"][0], x["v"][0], S, beta=x["beta"][0], a=x["a"][0],
                               r=x["r"][0], qn=x["qn"], p=C)
        for key in seen:
            seen[key].append(x[key][0][bi, hi])
        outs.append(o[bi, hi])
        ms.append(m[bi, hi])
    # sampled heads as a [1, 3, steps, d] scan for the oracle
    xs = {key: torch.stack(val, dim=1)[None] for key, val in seen.items()}
    xs["qn"] = w.qn
    ref = run_oracle(variant, xs)
    got = {"o": torch.stack(outs, dim=1)[None], "m": torch.stack(ms, dim=1)[None], "S": S[bi, hi][None]}
    if variant == "kalman_diag":
        got["p"] = C[bi, hi][None]
    compare(got, ref, TOL["bf16"])


# ----------------------------------------------------------------------------- status and errors


def test_numeric_status_flag_for_non_positive_innovation_variance():
    w = WORKLOADS["gdn_d64"].with_(variant="kalman_full")
    x = make_scan_inputs(w, seed=10, device=DEV, B=1, H=1, L=20)
    x["r"][0, 0, 5] = -10.0
    ws = torch.empty(kdn.workspace_bytes("kalman_full", 1, 1, 20, 64, 64), dtype=torch.uint8, device=DEV)
    kdn.scan_kalman_full(x["q"], x["k"], x["v"], x["r"], a=x["a"], qn=0.0, workspace=ws)
    assert kdn.read_device_status(ws) == kdn.KDN_ERR_NUMERIC
    x["r"][0, 0, 5] = 1.0
    kdn.scan_kalman_full(x["q"], x["k"], x["v"], x["r"], a=x["a"], qn=0.0, workspace=ws)
    assert kdn.read_device_status(ws) == kdn.KDN_OK


def test_isotropic_numeric_status_flag():
    w = WORKLOADS["gdn_d64"].with_(variant="kalman_iso")
    x = make_scan_inputs(w, seed=10, device=DEV, B=1, H=2, L=300)
    x["r"][0, 1, 250] = -10.0
    ws = torch.empty(kdn.workspace_bytes("kalman_iso", 1, 2, 300, 64, 64), dtype=torch.uint8, device=DEV)
    kdn.scan_kalman_iso(x["q"], x["k"], x["v"], x["r"], a=x["a"], qn=0.0, workspace=ws)
    assert kdn.read_device_status(ws) == kdn.KDN_ERR_NUMERIC
    x["r"][0, 1, 250] = 1.0
    kdn.scan_kalman_iso(x["q"], x["k"], x["v"], x["r"], a=x["a"], qn=0.0, workspace=ws)
    assert kdn.read_device_status(ws) == kdn.KDN_OK


def test_host_pointer_and_small_workspace_are_rejected():
    L = kdn.lib()
    w = WORKLOADS["gdn_d64"]
    x = make_scan_inputs(w, seed=11, device=DEV, B=1, H=1, L=8)
    S = torch.zeros(1, 1, 64, 64, device=DEV)
    o = torch.empty(1, 1, 8, 64, dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    host_S = torch.zeros(1, 1, 64, 64)
    d = kdn.Dims(1, 1, 8, 64, 64, 0, kdn.KDN_BF16, kdn.KDN_BF16)
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = L.kdn_scan_delta(ctypes.byref(d), p(x["q"]), p(x["k"]), p(x["v"]), p(x["beta"]), None, p(host_S), p(o), None,
                          p(ws), 256, None)
    assert st == kdn.KDN_ERR_INVALID_ARG
    st = L.kdn_scan_kalman_diag(ctypes.byref(d), p(x["q"]), p(x["k"]), p(x["v"]), None, p(x["r"]), None, 0.0, p(S),
                                p(torch.ones(1, 1, 64, device=DEV)), p(o), None, p(ws), 256, None)
    assert st == kdn.KDN_ERR_INVALID_ARG
    assert b"workspace" in L.kdn_last_error()


def test_nan_input_propagates_and_flags():
    w = WORKLOADS["gdn_d64"].with_(variant="kalman_diag", qn=1e-3)
    x = make_scan_inputs(w, seed=12, device=DEV, B=1, H=1, L=40)
    x["r"][0, 0, 10] = float("nan")
    ws = torch.empty(kdn.workspace_bytes("kalman_diag", 1, 1, 40, 64, 64), dtype=torch.uint8, device=DEV)
    o, m, S, p = kdn.scan_kalman_diag(x["q"], x["k"], x["v"], x["r"], a=x["a"], qn=1e-3, workspace=ws)
    assert kdn.read_device_status(ws) == kdn.KDN_ERR_NUMERIC
    assert torch.isnan(S).any()
