"""GPU parity of the surprise-cache read (A Hippocampus for Linear Attention, sections 3.3-3.4) against
the float64 oracle, through the C ABI.  The cache's token indices are integers: compared exactly (the
surprise values are continuous, so ties do not occur).  o within 1e-4 (fp32 inputs) / 3e-3 (bf16)."""

import numpy as np
import pytest
import torch

import oracle
from delta_rule_recurrent_scan_b200 import kdn
from delta_rule_recurrent_scan_b200.workloads import WORKLOADS, make_scan_inputs
from parity import TOL, normwise_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _params(dk, H, seed):
    g = torch.Generator().manual_seed(seed)
    gq = (0.5 + torch.rand(dk, generator=g)).to(DEV)
    gk = (0.5 + torch.rand(dk, generator=g)).to(DEV)
    sink = torch.randn(H, generator=g).to(DEV)
    return gq, gk, sink


def _np(t):
    return t.detach().double().cpu().numpy()


def _check(x, m, gq, gk, sink, w, block, tol, tokens=None, heads=None):
    o, cache = kdn.hola_cache_read(x["q"], x["k"], x["v"], m, gq, gk, sink, w=w, block=block)
    torch.cuda.synchronize()
    q, k, v, mm = _np(x["q"]), _np(x["k"]), _np(x["v"]), _np(m)
    if heads is not None:
        sel = lambda a: np.stack([a[b, h] for b, h in heads])[None]  # noqa: E731
        q, k, v, mm = sel(q), sel(k), sel(v), sel(mm)
        o = torch.stack([o[b, h] for b, h in heads])[None]
        cache = torch.stack([cache[b, h] for b, h in heads])[None]
        sink_np = np.array([_np(sink)[h] for _, h in heads])
    else:
        sink_np = _np(sink)
    ref = oracle.hola_cache_read(q, k, v, mm, _np(gq), _np(gk), sink_np, w=w, block=block, tokens=tokens)
    assert np.array_equal(cache.cpu().numpy(), ref["cache"])
    got = o if tokens is None else o[:, :, tokens]
    exp = ref["o"] if tokens is None else ref["o"][:, :, tokens]
    err = normwise_err(got, exp)
    assert err <= tol, err
    return err


@pytest.mark.parametrize("w,block", [(64, 64), (8, 64), (8, 16), (64, 32)])
def test_bf16_d128_several_blocks_and_evictions(w, block):
    wl = WORKLOADS["gdn_d128"]
    x = make_scan_inputs(wl, seed=1, device=DEV, B=1, H=2, L=300)
    m = torch.rand(1, 2, 300, device=DEV)
    gq, gk, sink = _params(128, 2, 0)
    _check(x, m, gq, gk, sink, w, block, TOL["bf16"])


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 16), (128, 32)])
def test_fp32_inputs_and_unequal_dims(dk, dv):
    wl = WORKLOADS["gdn_d64"].with_(dk=dk, dv=dv, dtype="f32")
    x = make_scan_inputs(wl, seed=2, device=DEV, B=2, H=2, L=150)
    m = torch.rand(2, 2, 150, device=DEV)
    gq, gk, sink = _params(dk, 2, 1)
    _check(x, m, gq, gk, sink, 16, 32, TOL["f32"])


def test_surprise_from_a_delta_scan_selects_the_cache():
    """The intended pipeline: m is the scan's own surprise output."""
    wl = WORKLOADS["gdn_d128"]
    x = make_scan_inputs(wl, seed=3, device=DEV, B=1, H=2, L=260)
    _, m, _ = kdn.scan_delta(x["q"], x["k"], x["v"], x["beta"], a=x["a"])
    gq, gk, sink = _params(128, 2, 2)
    _check(x, m, gq, gk, sink, 32, 64, TOL["bf16"])


def test_empty_and_single_token():
    wl = WORKLOADS["gdn_d64"]
    gq, gk, sink = _params(64, 2, 3)
    x = make_scan_inputs(wl, seed=4, device=DEV, B=1, H=2, L=1)
    _check(x, torch.rand(1, 2, 1, device=DEV), gq, gk, sink, 4, 64, TOL["bf16"])
    x0 = make_scan_inputs(wl, seed=4, device=DEV, B=1, H=2, L=0)
    o, cache = kdn.hola_cache_read(x0["q"], x0["k"], x0["v"], torch.rand(1, 2, 0, device=DEV), gq, gk, sink, w=4)
    torch.cuda.synchronize()
    assert o.numel() == 0 and bool((cache == -1).all())


def test_full_layer_sampled_heads_and_tokens():
    """The layer shape the benchmark times (B=8, H=16, L=8192, d=128), checked on sampled heads at
    tokens spread over the sequence (every block boundary case included)."""
    wl = WORKLOADS["gdn_d128"]
    x = make_scan_inputs(wl, seed=0, device=DEV)
    m = torch.rand(wl.B, wl.H, wl.L, device=DEV)
    gq, gk, sink = _params(128, wl.H, 4)
    tokens = [0, 1, 63, 64, 65, 127, 128, 1000, 4095, 4096, 8190, 8191]
    _check(x, m, gq, gk, sink, 64, 64, TOL["bf16"], tokens=tokens, heads=[(0, 0), (7, 15)])


@pytest.mark.parametrize("w,L", [(64, 300), (5, 700), (64, 64), (17, 1)])
def test_parallel_read_equals_the_block_by_block_walk(w, L):
    """With room for every block's cache indices the read runs all blocks at once; with the 256-byte status
    workspace one CTA per head walks them in order.  Same cache indices, o equal to fp32 rounding."""
    wl = WORKLOADS["gdn_d128"]
    x = make_scan_inputs(wl, seed=5, device=DEV, B=2, H=3, L=L)
    m = torch.rand(2, 3, L, device=DEV)
    m[0, 1, : L // 2] = 0.5  # ties in m: the earlier token wins in both forms
    gq, gk, sink = _params(128, 3, 2)
    small = torch.empty(256, dtype=torch.uint8, device=DEV)
    o_par, c_par = kdn.hola_cache_read(x["q"], x["k"], x["v"], m, gq, gk, sink, w=w)
    o_ser, c_ser = kdn.hola_cache_read(x["q"], x["k"], x["v"], m, gq, gk, sink, w=w, workspace=small)
    torch.cuda.synchronize()
    assert torch.equal(c_par, c_ser)
    assert normwise_err(o_par, _np(o_ser)) < 1e-5
    _check(x, m, gq, gk, sink, w, 64, TOL["bf16"])


@pytest.mark.parametrize("w,L", [(64, 64 * 192), (9, 64 * 193 - 5)])
def test_cache_scan_limit_and_the_walk_beyond_it(w, L):
    """Up to 192 blocks every block's cache comes from the log-depth scan over the blocks' ranked lists,
    beyond that from the serial walk over the blocks; both must give the caches (and o) of the block-by-block
    read, ties in m included."""
    wl = WORKLOADS["gdn_d128"]
    x = make_scan_inputs(wl, seed=6, device=DEV, B=1, H=2, L=L)
    m = torch.rand(1, 2, L, device=DEV)
    m[0, 1, : L // 3] = 0.25
    gq, gk, sink = _params(128, 2, 3)
    small = torch.empty(256, dtype=torch.uint8, device=DEV)
    o_par, c_par = kdn.hola_cache_read(x["q"], x["k"], x["v"], m, gq, gk, sink, w=w)
    o_ser, c_ser = kdn.hola_cache_read(x["q"], x["k"], x["v"], m, gq, gk, sink, w=w, workspace=small)
    torch.cuda.synchronize()
    assert torch.equal(c_par, c_ser)
    assert normwise_err(o_par, _np(o_ser)) < 1e-5
