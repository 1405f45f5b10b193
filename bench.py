#!/usr/bin/env python
"""Throughput of the gain-weighted residual memory scan on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl kdn|reference]

One step = one pass of the scan (every stage of the path: staging, gates,
gains, intra-chunk solves, output, state write-back) over one batch of
synthetic input resident in HBM.  The headline workload is the diagonal-Kalman
language-model layer (B=8, H=16, L=8192, d_k=d_v=128, bf16 inputs, fp32
state): the largest d=128 scan configuration.  The same line also reports the
other layer workloads (delta rule at d=128 and d=64, full Kalman at d=128) and
the decode step in ``also``.

Metric: scan tokens/s per layer (B*H*L / time).  Time is measured on the
device with CUDA events on the launching stream, after W warm-up steps, as the
max over ranks.  Inputs (about 1.1 GB per step) are larger than the 126 MB L2,
so no flush is needed between steps.

Multi-GPU (torchrun): every rank runs its own batch of the same shape (heads
are independent: weak scaling, no collective on the data path); the value is
the tokens all ranks processed divided by the slowest rank's time.

``--impl reference`` times the float64 CPU oracle on a bounded sample of the
same workload (rank 0 only) and prints the same line with "impl": "reference".
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from delta_rule_recurrent_scan_b200.workloads import WORKLOADS, make_decode_inputs, make_scan_inputs  # noqa: E402

HEADLINE = "kalman_diag_d128"
SECONDARY = ["gdn_d128", "kalman_iso_d128", "kalman_full_d128", "gdn_d64"]
DECODE = ["decode_delta", "decode_diag"]
METRIC = "scan tokens/s per layer (B*H*L/time) at d=128"


# ----------------------------------------------------------------------------- roofline bookkeeping


def algorithmic_bytes(w, in_bytes=2, out_bytes=4) -> int:
    """Bytes one scan must move: q, k, v in, o out, per-token scalars, m out, state in and out."""
    tok = w.B * w.H * w.L
    io = tok * ((2 * w.dk + w.dv) * in_bytes + w.dv * out_bytes + 4)  # + m
    scalars = {"delta": 8, "kalman_diag": 8, "kalman_full": 8, "kalman_iso": 8}[w.variant]  # beta|r and a
    state = w.B * w.H * w.dk * w.dv * 4 * 2
    if w.variant == "kalman_full":
        state += w.B * w.H * w.dk * w.dk * 4 * 2
    elif w.variant == "kalman_diag":
        state += w.B * w.H * w.dk * 4 * 2
    elif w.variant == "kalman_iso":
        state += w.B * w.H * 4 * 2
    return io + tok * scalars + state


def decode_bytes(w, in_bytes=2, out_bytes=4) -> int:
    n = w.B * w.H
    per = (2 * w.dk + w.dv) * in_bytes + w.dv * out_bytes + 4 + 8 + w.dk * w.dv * 4 * 2
    if w.variant == "kalman_diag":
        per += w.dk * 4 * 2
    return n * per


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the dominant kernel from one ncu
# capture, per token (it scales with the tokens of a launch).  Valid only for the kernel sources it was
# taken on: a different hash of those files reports null.
_WS_SOURCES = ["delta_rule_recurrent_scan_b200/csrc/chunk_scan_ws.cu",
               "delta_rule_recurrent_scan_b200/csrc/chunk_common.cuh",
               "delta_rule_recurrent_scan_b200/csrc/sm100.cuh",
               "delta_rule_recurrent_scan_b200/csrc/mobius.cuh"]
_RICCATI_SOURCES = ["delta_rule_recurrent_scan_b200/csrc/riccati.cu",
                    "delta_rule_recurrent_scan_b200/csrc/chunk_common.cuh",
                    "delta_rule_recurrent_scan_b200/csrc/sm100.cuh",
                    "delta_rule_recurrent_scan_b200/csrc/common.cuh"]
_B3 = 3 * 16 * 8192  # tokens of the reduced capture (B = 3 keeps one segment per head)
_WS_SHA = "913c18f440d3d0df7e31a9fe0288d4cc5e0a0097"
NCU_TRAFFIC = {
    "kalman_diag_d128": {"sources": _WS_SOURCES, "sha1": _WS_SHA,
                         "bytes_per_token": (308.486912e6 + 170.518272e6) / _B3,
                         "capture": "ncu, chunk_scan_ws_kernel<diag> at B=3 H=16 L=8192, per-token bytes scaled to the launch"},
    "gdn_d128": {"sources": _WS_SOURCES, "sha1": _WS_SHA,
                 "bytes_per_token": (308.391680e6 + 170.423808e6) / _B3,
                 "capture": "ncu, chunk_scan_ws_kernel<delta> at B=3 H=16 L=8192, per-token bytes scaled to the launch"},
    "kalman_iso_d128": {"sources": _WS_SOURCES, "sha1": _WS_SHA,
                        "bytes_per_token": (308.401664e6 + 172.895488e6) / _B3,
                        "capture": "ncu, chunk_scan_ws_kernel<iso> at B=3 H=16 L=8192, per-token bytes scaled to the launch"},
    "kalman_full_d128": {"sources": _RICCATI_SOURCES, "sha1": "c3a61774284b0bdb56eeaa3f4bd8987e544152b7",
                         "bytes_per_token": (31.137024e6 + 0.194560e6) / (2 * 8 * 4096),
                         "capture": "ncu, riccati_chain_tc_kernel at the full workload B=2 H=8 L=4096"},
}


def ncu_traffic(w):
    import hashlib

    rec = NCU_TRAFFIC.get(w.name)
    if rec is None:
        return None
    h = hashlib.sha1()
    try:
        for src in rec["sources"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
    except OSError:
        return None
    if h.hexdigest() != rec["sha1"]:
        return None
    return rec["bytes_per_token"] * w.tokens


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines: list[str] = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        mhz, max_mhz, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                mhz.append(float(parts[0]))
                max_mhz = float(parts[1])
            except ValueError:
                continue
            for name, val in zip(names, parts[3:7]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": max_mhz,
                "reasons": sorted(reasons), "samples": len(mhz)}


# ----------------------------------------------------------------------------- device timing


def _barrier(dist_on):
    if dist_on:
        torch.distributed.barrier()


def _max_over_ranks(x: float, dist_on: bool) -> float:
    """The slowest rank's value (NCCL groups reduce on the GPU, gloo groups on the CPU)."""
    if not dist_on:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(tokens_per_rank: int, ms_per_step: float, world: int) -> float:
    """Whole-job throughput: every rank runs its own batch of the same shape (independent heads);
    the job's time is the slowest rank's."""
    return tokens_per_rank * world / (ms_per_step * 1e-3)


def time_device(fn, steps, warmup, dist_on, clocks=None):
    """Mean ms per call of ``fn`` on the current stream, max over ranks."""
    for _ in range(warmup):
        fn()
    stream = torch.cuda.current_stream()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    _barrier(dist_on)
    ctx = clocks if clocks is not None else _NullCtx()
    with ctx:
        start.record(stream)
        for _ in range(steps):
            fn()
        end.record(stream)
        torch.cuda.synchronize()
    _barrier(dist_on)
    return _max_over_ranks(start.elapsed_time(end) / steps, dist_on)


class _NullCtx:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


# ----------------------------------------------------------------------------- workloads


def scan_closure(w, x, kdn):
    """A zero-argument step for workload ``w`` on resident inputs ``x``; returns (fn, outputs)."""
    B, H, dk, dv = w.B, w.H, w.dk, w.dv
    dev = x["q"].device
    S = torch.zeros(B, H, dk, dv, device=dev)
    o = torch.empty(B, H, w.L, dv, dtype=torch.float32, device=dev)
    m = torch.empty(B, H, w.L, device=dev)
    ws = torch.empty(kdn.workspace_bytes(w.variant, B, H, w.L, dk, dv), dtype=torch.uint8, device=dev)
    outs = {"o": o, "m": m, "S": S}
    if w.variant == "delta":
        def fn():
            kdn.scan_delta(x["q"], x["k"], x["v"], x["beta"], a=x["a"], S=S, o=o, m=m, workspace=ws)
        return fn, outs
    if w.variant == "kalman_full":
        P = torch.eye(dk, device=dev).repeat(B, H, 1, 1)
        outs["P"] = P

        def fn():
            kdn.scan_kalman_full(x["q"], x["k"], x["v"], x["r"], a=x["a"], qn=x["qn"], S=S, P=P, o=o, m=m,
                                 workspace=ws)
        return fn, outs
    if w.variant == "kalman_iso":
        c = torch.ones(B, H, device=dev)
        outs["c"] = c

        def fn():
            kdn.scan_kalman_iso(x["q"], x["k"], x["v"], x["r"], a=x["a"], qn=x["qn"], S=S, c=c, o=o, m=m,
                                workspace=ws)
        return fn, outs
    p = torch.ones(B, H, dk, device=dev)
    outs["p"] = p

    def fn():
        kdn.scan_kalman_diag(x["q"], x["k"], x["v"], x["r"], a=x["a"], qn=x["qn"], S=S, p=p, o=o, m=m, workspace=ws)
    return fn, outs


def scan_plan(w):
    from delta_rule_recurrent_scan_b200 import kdn
    return kdn.plan(w.variant, w.B, w.H, w.L, w.dk, w.dv,
                    in_dtype=torch.bfloat16 if w.dtype == "bf16" else torch.float32)


def bench_scan(w, steps, warmup, dist_on, rank, world, clocks=None):
    from delta_rule_recurrent_scan_b200 import kdn
    x = make_scan_inputs(w, seed=rank, device="cuda")
    fn, _ = scan_closure(w, x, kdn)
    ms = time_device(fn, steps, warmup, dist_on, clocks)
    return {"ms": ms, "value": weak_scaling_value(w.tokens, ms, world), "launches": scan_plan(w)["launches"] * steps}


# the per-token inputs each variant reads (Qn is a scalar argument)
E2E_INPUTS = {"delta": ("q", "k", "v", "beta", "a"), "kalman_full": ("q", "k", "v", "a", "r"),
              "kalman_diag": ("q", "k", "v", "a", "r"), "kalman_iso": ("q", "k", "v", "a", "r")}


def bench_e2e(w, steps, warmup, dist_on, rank, world):
    """Through the public API with host buffers, as a stream of batches: every step copies the inputs its
    variant reads from pinned host memory to the device, scans them and copies o, m and the final state
    (S and P, p or c) back.  Steps are pipelined over three streams with two device buffer sets, so that
    step i + 1's host-to-device copy runs beside step i's scan and device-to-host copy (the link is full
    duplex); the time per step is the span of all steps / steps."""
    from delta_rule_recurrent_scan_b200 import kdn
    xd = make_scan_inputs(w, seed=rank, device="cuda")
    keys = E2E_INPUTS[w.variant]
    host = {k: xd[k].cpu().pin_memory() for k in keys if isinstance(xd[k], torch.Tensor)}
    bufs = []
    for _ in range(2):
        dev = {k: (torch.empty_like(v) if isinstance(v, torch.Tensor) else v) for k, v in xd.items()}
        fn_dev, outs = scan_closure(w, dev, kdn)
        bufs.append((dev, fn_dev, outs))
    del xd
    out_host = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in bufs[0][2].items()}
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = sum(v.numel() * v.element_size() for v in out_host.values())

    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = {name: [torch.cuda.Event() for _ in range(2)] for name in ("in", "comp", "out")}
    cur = torch.cuda.current_stream()
    for name in ev:
        for e in ev[name]:
            e.record(cur)

    def step(i):
        b = i % 2
        dev, fn_dev, outs = bufs[b]
        s_in.wait_event(ev["comp"][b])       # the scan of step i - 2 has read these inputs
        with torch.cuda.stream(s_in):
            for k, v in host.items():
                dev[k].copy_(v, non_blocking=True)
            ev["in"][b].record(s_in)
        s_comp.wait_event(ev["in"][b])
        s_comp.wait_event(ev["out"][b])      # step i - 2's outputs are back on the host
        with torch.cuda.stream(s_comp):
            fn_dev()
            ev["comp"][b].record(s_comp)
        s_out.wait_event(ev["comp"][b])
        with torch.cuda.stream(s_out):
            for k, v in out_host.items():
                v.copy_(outs[k], non_blocking=True)
            ev["out"][b].record(s_out)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    _barrier(dist_on)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(cur)
    for st in (s_in, s_comp, s_out):
        st.wait_event(start)
    for i in range(steps):
        step(warmup + i)
    for st in (s_in, s_comp, s_out):
        cur.wait_stream(st)
    end.record(cur)
    torch.cuda.synchronize()
    _barrier(dist_on)
    ms = _max_over_ranks(start.elapsed_time(end) / steps, dist_on)
    return {"value": w.tokens * world / (ms * 1e-3), "ms": ms, "h2d": h2d, "d2h": d2h,
            "copied": {"in": list(host), "out": list(out_host)},
            "pipelined": "3 streams, 2 device buffer sets: step i + 1's copy-in beside step i's scan and copy-out"}


def bench_decode(w, steps, warmup, dist_on, rank, world):
    from delta_rule_recurrent_scan_b200 import kdn
    n_inputs = 8  # distinct token batches cycled through (inputs are per call; the 512 MB state dominates)
    x = make_decode_inputs(w, steps=n_inputs, seed=rank, device="cuda")
    S = torch.zeros(w.B, w.H, w.dk, w.dv, device="cuda")
    p = torch.ones(w.B, w.H, w.dk, device="cuda")
    o = torch.empty(w.B, w.H, w.dv, dtype=torch.float32, device="cuda")
    m = torch.empty(w.B, w.H, device="cuda")
    it = [0]

    def fn():
        t = it[0] % n_inputs
        it[0] += 1
        kdn.decode_step(w.variant, x["q"][t], x["k"][t], x["v"][t], S, beta=x["beta"][t], a=x["a"][t], r=x["r"][t],
                        qn=x["qn"], p=p if w.variant == "kalman_diag" else None, o=o, m=m)
    ms = time_device(fn, steps, warmup, dist_on)
    return {"ms": ms, "value": w.B * w.H * world / (ms * 1e-3), "launches": steps}


def bench_hola(w, steps, warmup, dist_on, rank, world, cache_w=64):
    """Surprise-cache read over a layer (the scan's m as the surprise; random here)."""
    from delta_rule_recurrent_scan_b200 import kdn
    x = make_scan_inputs(w, seed=rank, device="cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(rank)
    m = torch.rand(w.B, w.H, w.L, device="cuda", generator=g)
    gq = torch.ones(w.dk, device="cuda")
    gk = torch.ones(w.dk, device="cuda")
    sink = torch.zeros(w.H, device="cuda")
    o = torch.empty(w.B, w.H, w.L, w.dv, device="cuda")
    cache = torch.empty(w.B, w.H, cache_w, dtype=torch.int32, device="cuda")

    def fn():
        kdn.hola_cache_read(x["q"], x["k"], x["v"], m, gq, gk, sink, w=cache_w, block=64, o=o, cache=cache)
    ms = time_device(fn, steps, warmup, dist_on)
    # the cache choice and the block reads (bf16, d = 128); one block-by-block kernel elsewhere
    per_call = 2 if w.dtype == "bf16" and w.dk == 128 and w.dv == 128 else 1
    return {"ms": ms, "value": w.tokens * world / (ms * 1e-3), "launches": per_call * steps}


def bench_backward(w, steps, warmup, dist_on, rank, world):
    """The backward over a layer (gated delta rule; isotropic, diagonal or full Kalman: the memory backward with
    the uncertainty chain around it); upstream dO and dm random, start state zero."""
    from delta_rule_recurrent_scan_b200 import kdn
    x = make_scan_inputs(w, seed=rank, device="cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(rank + 1)
    dO = torch.randn(w.B, w.H, w.L, w.dv, device="cuda", generator=g)
    dm = torch.randn(w.B, w.H, w.L, device="cuda", generator=g)
    dims = kdn.Dims(w.B, w.H, w.L, w.dk, w.dv, 0, kdn.KDN_BF16, kdn.KDN_F32, 0)
    ws = torch.empty(int(kdn.lib().kdn_backward_workspace_bytes(kdn.VARIANTS[w.variant], dims)), dtype=torch.uint8,
                     device="cuda")

    def fn():
        if w.variant == "kalman_iso":
            kdn.scan_kalman_iso_backward(x["q"], x["k"], x["v"], x["r"], dO, a=x["a"], qn=x["qn"], dm=dm, workspace=ws)
        elif w.variant == "kalman_diag":
            kdn.scan_kalman_diag_backward(x["q"], x["k"], x["v"], x["r"], dO, a=x["a"], qn=x["qn"], dm=dm, workspace=ws)
        elif w.variant == "kalman_full":
            kdn.scan_kalman_full_backward(x["q"], x["k"], x["v"], x["r"], dO, a=x["a"], qn=x["qn"], dm=dm, workspace=ws)
        else:
            kdn.scan_delta_backward(x["q"], x["k"], x["v"], x["beta"], dO, a=x["a"], dm=dm, workspace=ws)
    ms = time_device(fn, steps, warmup, dist_on)
    return {"ms": ms, "value": w.tokens * world / (ms * 1e-3), "launches": (2 if w.variant == "delta" else 4) * steps}


def backward_bytes(w, in_bytes=2) -> int:
    """q, k, v, beta, a, dO, dm in; dq, dk, dv, dbeta, da out (fp32)."""
    return w.tokens * ((2 * w.dk + w.dv) * in_bytes + 8 + w.dv * 4 + 4 + (2 * w.dk + w.dv) * 4 + 8)


def backward_flops(w, C=32) -> int:
    """Multiply-adds of the chunked backward (forward recompute included) per token: 8 d^2 + 11 C d, times 2; the
    full-covariance side adds 10 d^2 (forward and block recompute: a matrix-vector product and a rank-1 update each;
    backward: four matrix-vector products and the rank-2 update of the adjoint)."""
    d = w.dk
    return w.tokens * 2 * (8 * d * d + 11 * C * d + (10 * d * d if w.variant == "kalman_full" else 0))


FP32_CUDA_CORE_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # 148 SMs x 128 fp32 FMA lanes at 1965 MHz


def hola_bytes(w, in_bytes=2) -> int:
    """q, k, v in, m in, o^cache out (fp32), the final cache indices."""
    return w.tokens * ((2 * w.dk + w.dv) * in_bytes + 4 + w.dv * 4) + w.B * w.H * 64 * 4


# ----------------------------------------------------------------------------- CPU baseline (oracle)


def _oracle_head(args):
    """One head of the workload through the float64 oracle, as it stands (runs in a pool worker).
    Returns (tokens, seconds of the oracle call alone)."""
    name, overrides, seed = args
    import oracle

    w = WORKLOADS[name].with_(**overrides)
    x = make_scan_inputs(w, seed=seed, device="cpu", B=1, H=1)
    np_ = {k: (v.double().numpy() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    t0 = time.perf_counter()
    if w.variant == "delta":
        oracle.scan_delta(np_["q"], np_["k"], np_["v"], np_["beta"], a=np_["a"])
    elif w.variant == "kalman_full":
        oracle.scan_kalman_full(np_["q"], np_["k"], np_["v"], r=np_["r"], a=np_["a"], qn=np_["qn"])
    elif w.variant == "kalman_iso":
        oracle.scan_kalman_iso(np_["q"], np_["k"], np_["v"], r=np_["r"], a=np_["a"], qn=np_["qn"])
    else:
        oracle.scan_kalman_diag(np_["q"], np_["k"], np_["v"], r=np_["r"], a=np_["a"], qn=np_["qn"])
    return w.L, time.perf_counter() - t0


def _pool_init():
    torch.set_num_threads(1)
    import oracle  # noqa: F401  (import cost outside the timed calls)


class OraclePool:
    """The oracle on every host core: a spawn pool (safe beside a CUDA context) of one single-threaded
    worker per core in this process's affinity mask; heads are independent, so each worker scans whole
    heads.  Throughput = the tokens of one round (one head per worker) / the slowest worker's oracle time."""

    def __init__(self):
        import concurrent.futures
        import multiprocessing

        self.cores = len(os.sched_getaffinity(0))
        for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
            os.environ[var] = "1"  # one thread per worker process; the workers cover the cores
        self.pool = concurrent.futures.ProcessPoolExecutor(
            max_workers=self.cores, mp_context=multiprocessing.get_context("spawn"), initializer=_pool_init)

    def round(self, w, seed0=0):
        over = {"B": w.B, "H": w.H}
        res = list(self.pool.map(_oracle_head, [(w.name, over, seed0 + i) for i in range(self.cores)]))
        tokens = sum(r[0] for r in res)
        return tokens, max(r[1] for r in res)

    def close(self):
        self.pool.shutdown()


def cpu_baseline(w):
    """The float64 oracle, as it stands, on a bounded sample of the workload on all host cores."""
    pool = OraclePool()
    try:
        pool.round(w.with_(L=64), seed0=10_000)  # start the workers (spawn, imports) outside the timing
        tokens, dt = pool.round(w)
    finally:
        pool.close()
    return {"value": tokens / dt, "unit": "tokens/s", "cores": pool.cores, "kind": "oracle",
            "sample": f"{pool.cores} of {w.B * w.H} heads x full L={w.L} ({tokens} tokens), one head per worker "
                      f"on {pool.cores} single-threaded spawn workers (one per core), float64 NumPy, "
                      f"slowest worker {dt:.2f} s"}


# ----------------------------------------------------------------------------- main


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="kdn", choices=["kdn", "reference"])
    ap.add_argument("--no-also", action="store_true", help="skip the secondary workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurement")
    ap.add_argument("--batch", type=int, default=None, help="override B of the workload (profiling runs)")
    ap.add_argument("--backward-only", action="store_true",
                    help="time only the backward of a gated-delta or Kalman workload (profiling runs): one JSON line")
    ap.add_argument("--cache-read-only", action="store_true",
                    help="time only the surprise-cache read over a workload's shape (profiling runs): one JSON line")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = WORKLOADS[args.workload]
    if args.batch is not None:
        w = w.with_(B=args.batch)

    if args.impl == "reference":
        return reference_arm(args, w, rank, world)

    torch.cuda.set_device(local)
    dist_on = world > 1
    if dist_on:
        import datetime

        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))

    from delta_rule_recurrent_scan_b200 import kdn

    kdn.lib()  # fail loudly if the library is missing
    peak, peak_kind = measured_peaks()
    if args.cache_read_only:
        r = bench_hola(w, args.steps, args.warmup, dist_on, rank, world)
        if rank == 0:
            print(json.dumps({"metric": "surprise-cache read tokens/s (w = 64, blocks of 64)", "value": r["value"],
                              "unit": "tokens/s", "ms_per_step": r["ms"], "steps": args.steps,
                              "warmup": args.warmup, "gpu_launches": r["launches"],
                              "config": {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "dk": w.dk}}),
                  flush=True)
        if dist_on:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        return
    if args.backward_only:
        if w.variant not in ("delta", "kalman_iso", "kalman_diag", "kalman_full"):
            raise SystemExit("--backward-only needs a gated-delta or Kalman workload")
        r = bench_backward(w, args.steps, args.warmup, dist_on, rank, world)
        if rank == 0:
            print(json.dumps({"metric": f"{w.variant} backward tokens/s (every input gradient)", "value": r["value"],
                              "unit": "tokens/s", "ms_per_step": r["ms"], "steps": args.steps,
                              "warmup": args.warmup, "gpu_launches": r["launches"],
                              "config": {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "dk": w.dk}}),
                  flush=True)
        if dist_on:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        return
    clocks = ClockSampler(local)
    head = bench_scan(w, args.steps, args.warmup, dist_on, rank, world, clocks=clocks)
    ms = head["ms"]
    alg = algorithmic_bytes(w)
    achieved = alg / (ms * 1e-3) / 1e9
    plan = scan_plan(w)
    torch.cuda.empty_cache()

    e2e = None if args.no_e2e else bench_e2e(w, min(args.steps, 10), 3, dist_on, rank, world)
    torch.cuda.empty_cache()

    also = []
    if not args.no_also:
        for name in SECONDARY:
            if name == args.workload:
                continue
            sw = WORKLOADS[name]
            r = bench_scan(sw, max(3, args.steps // 4), 3, dist_on, rank, world)
            ab = algorithmic_bytes(sw)
            also.append({"workload": name, "variant": sw.variant, "value": r["value"], "unit": "tokens/s",
                         "ms_per_step": r["ms"], "gpu_launches": r["launches"],
                         "roofline_frac": ab / (r["ms"] * 1e-3) / 1e9 / peak})
            del r
            torch.cuda.empty_cache()
        hw = WORKLOADS["gdn_d128"]
        r = bench_hola(hw, max(3, args.steps // 4), 3, dist_on, rank, world)
        ab = hola_bytes(hw)
        also.append({"workload": "hola_cache_read_d128", "variant": "surprise-cache read (w=64, block 64)",
                     "value": r["value"], "unit": "tokens/s", "ms_per_step": r["ms"], "gpu_launches": r["launches"],
                     "roofline_frac": ab / (r["ms"] * 1e-3) / 1e9 / peak})
        del r
        torch.cuda.empty_cache()
        for bname, bvariant in (("gdn_d128", "delta backward (dq, dk, dv, dbeta, da, dS0)"),
                                ("kalman_iso_d128", "isotropic Kalman backward (dq, dk, dv, dr, da, dqn, dS0, dc0)"),
                                ("kalman_diag_d128", "diagonal Kalman backward (dq, dk, dv, dr, da, dqn, dS0, dp0)"),
                                ("kalman_full_d128", "full Kalman backward (dq, dk, dv, dr, da, dqn, dS0, dP0)")):
            bw = WORKLOADS[bname]
            r = bench_backward(bw, 2, 3, dist_on, rank, world)
            also.append({"workload": bname + "_backward", "variant": bvariant,
                         "value": r["value"], "unit": "tokens/s", "ms_per_step": r["ms"], "gpu_launches": r["launches"],
                         "roofline_frac": backward_bytes(bw) / (r["ms"] * 1e-3) / 1e9 / peak,
                         "fp32_flop_frac": backward_flops(bw) / (r["ms"] * 1e-3) / 1e12 / FP32_CUDA_CORE_TFLOPS,
                         "arith": "f32 CUDA cores"})
            del r
            torch.cuda.empty_cache()
        for name in DECODE:
            dw = WORKLOADS[name]
            r = bench_decode(dw, 64, 8, dist_on, rank, world)
            ab = decode_bytes(dw)
            also.append({"workload": name, "variant": dw.variant, "value": r["value"], "unit": "states/s",
                         "ms_per_step": r["ms"], "gpu_launches": r["launches"],
                         "roofline_frac": ab / (r["ms"] * 1e-3) / 1e9 / peak})
            torch.cuda.empty_cache()

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": head["value"],
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16" if plan["arith"] == "bf16-tc" else "f32",
            "data": "synthetic",
            "config": {"workload": w.name, "variant": w.variant, "B": w.B, "H": w.H, "L": w.L, "dk": w.dk,
                       "dv": w.dv, "in_dtype": w.dtype, "out_dtype": "f32", "state": "fp32", "seed": "rank",
                       "l2": f"inputs larger than L2 ({alg / 1e9:.2f} GB per step), no flush",
                       "parallelism": f"dp{world} (independent heads, no collective)",
                       "kernel_path": plan},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": ncu_traffic(w), "peak_source": peak_kind,
                         "algorithmic_bytes_per_launch": alg, "kernel": plan["kernel"],
                         "timed": "whole C-ABI call (status-word memset + kernels) with CUDA events",
                         # the same time against the bytes of a bf16 read-out (the figure the per-token
                         # byte table of the method's roofline uses; this scan writes o in fp32)
                         "frac_bf16_o_bytes": algorithmic_bytes(w, out_bytes=2) / (ms * 1e-3) / 1e9 / peak,
                         "algorithmic_bytes_bf16_o_per_launch": algorithmic_bytes(w, out_bytes=2)},
            "e2e": None if e2e is None else {"value": e2e["value"], "unit": "tokens/s",
                                             "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                                             "ms_per_step": e2e["ms"], "copied": e2e["copied"],
                                             "pipelined": e2e["pipelined"]},
            "gpu_launches": head["launches"],
            "clocks": clocks.summary(),
            "also": also,
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def reference_arm(args, w, rank, world):
    """The float64 CPU oracle as the reference arm: rank 0 only; each step is one round of the oracle
    pool (one head of the workload per host core, full L)."""
    if rank != 0:
        return
    pool = OraclePool()
    try:
        pool.round(w.with_(L=64), seed0=10_000)  # start the workers outside the timing
        for i in range(min(args.warmup, 1)):
            pool.round(w, seed0=100 * (i + 1))
        total_tokens, total_s = 0, 0.0
        for i in range(args.steps):
            tokens, dt = pool.round(w, seed0=i * pool.cores)
            total_tokens += tokens
            total_s += dt
    finally:
        pool.close()
    dt = total_s / args.steps
    value = total_tokens / total_s
    sample = (f"{pool.cores} of {w.B * w.H} heads x full L={w.L} per step ({total_tokens // args.steps} tokens), "
              f"one head per single-threaded spawn worker, {pool.cores} workers (one per core), float64 NumPy")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "variant": w.variant, "B": w.B, "H": w.H, "L": w.L, "dk": w.dk, "dv": w.dv},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": pool.cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
