"""The multi-rank path of bench.py on CPU with two gloo ranks: every rank runs its
own replica on its own token shard (same expert weights), the job time is the
slowest rank's, and the job value counts every rank's tokens.  No GPU, no data
collective on the layer itself -- only the timing reduction."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from combine_overlap_b200 import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        times = [1.0 + rank, 5.0 - rank, 2.5]          # ms, per rank
        got = bench.max_over_ranks(times, world)
        wl = synth.WORKLOADS["tiny"]
        x, logits, W1, W3, W2 = bench.rank_inputs(wl, rank)
        xs = [torch.zeros_like(x, dtype=torch.float32) for _ in range(world)]
        dist.all_gather(xs, x.float().contiguous())
        ws = [torch.zeros_like(W1, dtype=torch.float32) for _ in range(world)]
        dist.all_gather(ws, W1.float().contiguous())
        out[rank] = dict(got=got, same_weights=all(torch.equal(ws[0], w) for w in ws),
                         distinct_tokens=not torch.equal(xs[0], xs[1]),
                         value=bench.job_tokens_per_s(wl.T, world, got[0]))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_and_max_timing():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        res = out[r]
        assert res["got"] == [2.0, 5.0, 2.5]            # element-wise max over ranks
        assert res["same_weights"] and res["distinct_tokens"]
        assert res["value"] == pytest.approx(256 * 2 / 2.0e-3)


def test_single_rank_is_identity():
    assert bench.max_over_ranks([3.0, 4.0], 1) == [3.0, 4.0]
    assert bench.shard_workload(synth.WORKLOADS["tiny"], 0) is synth.WORKLOADS["tiny"]
