"""The multi-GPU bench path on CPU: two gloo ranks, no GPU.

The scan shards by heads with no data-path collective (every rank runs its own
batch of the same shape); the only cross-rank steps are the barriers around the
timed region and the max over ranks of the step time.  This checks that logic
with world_size 2 over gloo on 127.0.0.1.
"""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    from delta_rule_recurrent_scan_b200.workloads import WORKLOADS, make_scan_inputs

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        # each rank times a different amount: the job takes the slowest
        ms = bench._max_over_ranks(1.0 + rank, True)
        w = WORKLOADS["kalman_diag_d128"]
        value = bench.weak_scaling_value(w.tokens, ms, world)
        # ranks draw different (seeded) inputs of the same shape
        x = make_scan_inputs(w.with_(B=1, H=1, L=8), seed=rank)
        first = float(x["v"].flatten()[0])
        vals = [torch.zeros(1) for _ in range(world)]
        dist.all_gather(vals, torch.tensor([first]))
        out[rank] = (ms, value, [float(v) for v in vals])
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_and_weak_scale():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=240)
            assert p.exitcode == 0
        res = dict(out)
    from delta_rule_recurrent_scan_b200.workloads import WORKLOADS

    tokens = WORKLOADS["kalman_diag_d128"].tokens
    for r in range(world):
        ms, value, firsts = res[r]
        assert ms == pytest.approx(2.0)  # max over ranks
        assert value == pytest.approx(tokens * world / 2.0e-3)
        assert firsts[0] != firsts[1]  # independent shards
