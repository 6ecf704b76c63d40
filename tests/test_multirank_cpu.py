"""Multi-rank host logic on CPU: two gloo ranks, one microbatch each.

The path has no collective: each rank builds its own candidate set from its
own microbatch, with its window staggered by V * rank // world
(sampled_softmax.py, CandidateBuilder.reset). The oracle stands in for the
device here; the checks are on the per-rank plumbing the benchmark uses:
distinct seeds and offsets, different negatives per rank, the max-over-ranks
timing reduction, and the data-parallel gradient sync of the dense dW that
follows the path (ranks.allreduce_dw, the call the benchmark makes over NCCL).
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


# ------------------------------------------- data-parallel dW gradient sync --

def _dp_worker(rank, world, port, out_dir):
    """Each rank: its own microbatch through the oracle, dW rounded to bf16 as
    the device writes it, then ranks.allreduce_dw over gloo."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    T, d, V, P = 400, 16, 3001, 700
    off = ranks.rank_offset(123, V, rank, world)
    x_bits, lm_bits, targets = wl.make_inputs(T, d, V, 1.1, 0.05, ranks.rank_seed(9, rank))
    o = oc.sampled_ce(wl.bits_to_f64(x_bits), wl.bits_to_f64(lm_bits), targets, P, off)
    mine = torch.from_numpy(o["dW"]).to(torch.bfloat16)
    summed = mine.clone()
    ranks.allreduce_dw(summed, dist)
    np.savez(os.path.join(out_dir, f"dp{rank}.npz"), cand=o["candidates"], dW64=o["dW"],
             mine=mine.view(torch.int16).numpy(), summed=summed.view(torch.int16).numpy())
    dist.barrier()
    dist.destroy_process_group()


def test_dp_allreduce_of_dw_two_gloo_ranks(tmp_path):
    """The data-parallel sync sums the ranks' dense dW: rows in the union of the
    ranks' candidate sets carry the sum of their contributions, every other row
    stays +0.0 bit for bit, and all ranks end with the same tensor."""
    world = 2
    mp.start_processes(_dp_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    r = [np.load(tmp_path / f"dp{i}.npz") for i in range(world)]
    assert np.array_equal(r[0]["summed"], r[1]["summed"])
    bits = r[0]["summed"].view(np.uint16)
    V = bits.shape[0]
    union = np.zeros(V, bool)
    for k in range(world):
        union[r[k]["cand"]] = True
    assert np.all(bits[~union] == 0)                          # +0.0 outside the union
    got = wl.bits_to_f64(bits)
    mine = [wl.bits_to_f64(r[k]["mine"].view(np.uint16)) for k in range(world)]
    # two bf16 addends: the sum rounded once to bf16
    want_bf16 = wl.bits_to_f64(wl.bf16_bits((mine[0] + mine[1]).astype(np.float32)))
    assert np.array_equal(got, want_bf16)
    # and within the gradient tolerance of the float64 sum of the ranks' gradients
    exact = r[0]["dW64"] + r[1]["dW64"]
    assert np.linalg.norm(got - exact) <= 2e-2 * np.linalg.norm(exact)
    both = np.intersect1d(r[0]["cand"], r[1]["cand"])
    assert both.size > 0 and np.any(np.abs(got[both] - mine[0][both]) > 0)
    only0 = np.setdiff1d(r[0]["cand"], r[1]["cand"])
    assert np.array_equal(got[only0], mine[0][only0])        # one contribution: unchanged
