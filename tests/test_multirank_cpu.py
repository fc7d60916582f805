"""The multi-GPU bench path on CPU: two gloo ranks, sharding and timing logic.

Batch elements are independent, so the only cross-rank steps are the timing
barrier and the max-over-ranks of the device time; the inputs of a rank's
slice are the same elements a single process would generate for a bigger
batch (per-element seeds), so N ranks together run one weak-scaled job.
"""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from sparse_spd_selected_b200 import inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        elems = bench.shard_elements(rank, 3)
        g = inputs.chain_inputs(6, 5, 4, seed=9, load=1.0, elements=elems)[0]
        fake_ms = 10.0 + 5.0 * rank                       # rank 1 is the slow one
        ms = bench.max_over_ranks(fake_ms, world)
        dist.barrier()
        out[rank] = (elems, g.sum(), ms, bench.job_throughput(world, 3 * 5, 4, ms))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_time():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == [0, 1, 2] and res[1][0] == [3, 4, 5]     # disjoint contiguous slices
    full = inputs.chain_inputs(6, 5, 4, seed=9, load=1.0)[0]      # one process, whole batch
    assert np.isclose(res[0][1], full[:3].sum()) and np.isclose(res[1][1], full[3:].sum())
    assert res[0][2] == res[1][2] == 15.0                         # the slowest rank's time
    assert res[0][3] == pytest.approx(2 * 15 * 4 / 0.015)         # all ranks' blocks / job time


def test_single_rank_helpers():
    assert bench.shard_elements(0, 4) == [0, 1, 2, 3]
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.job_throughput(1, 100, 2, 1000.0) == 200.0
