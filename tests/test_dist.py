"""The multi-GPU host logic on CPU: two gloo ranks, distinct per-rank batches, the
max-over-ranks time and the whole-job throughput the benchmark reports."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_deltanet_mixer_verify_b200.dist import (max_over_ranks, rank_seed,
                                                    weak_scaling_throughput)
from gated_deltanet_mixer_verify_b200.inputs import make_inputs, workload


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = workload("batched_verify", B=2, seed=rank_seed(1002, rank))
        x = make_inputs(w)
        # every rank reports a different "time"; all must agree on the max
        t = max_over_ranks(0.010 * (rank + 1))
        # gather the first q element of each rank to check the batches differ
        first = torch.tensor([float(x["q"].float()[0, 0, 0, 0])])
        allf = [torch.zeros(1) for _ in range(world)]
        dist.all_gather(allf, first)
        q.put((rank, t, [float(f) for f in allf]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, firsts in out:
        assert t == pytest.approx(0.020)
        assert firsts[0] != firsts[1]


def test_single_process_identity_and_throughput():
    assert max_over_ranks(0.5) == 0.5
    assert rank_seed(1002, 0) == 1002 and rank_seed(1002, 3) == 1002 + 3 * 7919
    assert weak_scaling_throughput(100.0, 4, 2.0) == 200.0
    with pytest.raises(ValueError):
        weak_scaling_throughput(1.0, 1, 0.0)
