"""Multi-rank host logic on CPU: two gloo ranks, one microbatch each.

The path has no collective: each rank builds its own candidate set from its
own microbatch, with its window staggered by V * rank // world
(sampled_softmax.py, CandidateBuilder.reset). The oracle stands in for the
device build here; the checks are on the per-rank plumbing the benchmark
uses: distinct seeds and offsets, different negatives per rank, and the
max-over-ranks timing reduction.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import sampled_ce as oc
from sampled_softmax_cross_b200 import ranks
from sampled_softmax_cross_b200 import workloads as wl


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    V, P, T = 50304, 4096, 2000
    off = ranks.rank_offset(22656, V, rank, world)
    _, _, targets = wl.make_inputs(T, 8, V, 1.05, 0.01, ranks.rank_seed(3, rank))
    cand, tpos, vpos, info = oc.build_candidates(targets, V, P, off)
    # per-rank "time": the max over ranks must be the larger one
    t_max = ranks.max_over_ranks(10.0 + rank, dist)
    offs = [None] * world
    dist.all_gather_object(offs, off)
    np.savez(os.path.join(out_dir, f"r{rank}.npz"), cand=cand, off=off, t_max=t_max,
             offs=np.array(offs), need=info["need"], draw=info["draw"])
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    r = [np.load(tmp_path / f"r{i}.npz") for i in range(world)]
    V = 50304
    assert int(r[0]["off"]) == 22656 and int(r[1]["off"]) == (22656 + V // 2) % V
    assert list(r[0]["offs"]) == list(r[1]["offs"])
    assert float(r[0]["t_max"]) == 11.0 and float(r[1]["t_max"]) == 11.0
    # different microbatches and windows -> different candidate sets
    assert not np.array_equal(r[0]["cand"], r[1]["cand"])
    # the windows of the two ranks do not overlap here (draw < V / 2)
    for i in range(world):
        assert int(r[i]["draw"]) < V // 2


def test_rank_offset_and_seed():
    assert [ranks.rank_offset(0, 50304, k, 8) for k in range(8)] == [50304 * k // 8 for k in range(8)]
    assert ranks.rank_offset(50000, 50304, 1, 2) == (50000 + 25152) % 50304
    assert ranks.rank_seed(3, 2) == 5
    assert ranks.max_over_ranks(4.5, None) == 4.5
