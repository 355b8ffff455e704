"""The bench's multi-rank path (one process per GPU) on CPU: two gloo ranks
run the same cross-rank steps bench.py takes between its timed regions."""
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from test_sequence_layers_layer_b200 import synth  # noqa: E402


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        wl = synth.WORKLOADS["linear_ln_d64_b8h12_t2048"]
        mine = bench.rank_workload(wl, rank)
        # each rank's own inputs
        inp = synth.make_inputs(mine.scaled(B=1, H=1, T=32))
        sig = torch.tensor([float(inp.Q[0, 0, 0, 0]), float(mine.seed)])
        sigs = [torch.zeros(2) for _ in range(world)]
        dist.all_gather(sigs, sig)
        # rank r measured (10 + r) ms over 4 steps, e2e (20 - r) ms, 4 + r launches
        total, e2e, launches = bench.reduce_across_ranks(10.0 + rank, 20.0 - rank, 4 + rank, world,
                                                         torch.device("cpu"))
        tokens, ms_step, value = bench.aggregate(wl, world, 4, total)
        out[rank] = (tuple(float(v) for s in sigs for v in s), total, e2e, launches, tokens, ms_step,
                     value)
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_and_shard():
    world, port = 2, 29500 + os.getpid() % 1000
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    wl = synth.WORKLOADS["linear_ln_d64_b8h12_t2048"]
    sigs0, total0, e2e0, l0, tok0, ms0, v0 = res[0]
    assert res[1][1:] == res[0][1:]          # every rank ends with the same job figures
    assert total0 == 11.0 and e2e0 == 20.0   # slowest rank (MAX)
    assert l0 == 4 + 5                        # launches summed over ranks
    assert tok0 == 2 * wl.tokens
    assert ms0 == pytest.approx(11.0 / 4)
    assert v0 == pytest.approx(2 * wl.tokens * 4 / 11e-3)
    # seeds differ by rank, and so do the inputs (weak scaling, disjoint data)
    assert sigs0[1] == wl.seed and sigs0[3] == wl.seed + 1
    assert sigs0[0] != sigs0[2]


def test_single_rank_is_identity():
    assert bench.reduce_across_ranks(3.0, 4.0, 5, 1, None) == (3.0, 4.0, 5)
