"""The multi-rank path on the CPU: two gloo ranks shard the batch (one seed
per rank), compute the operator's gradients with the oracle as a stand-in for
the device, and sum the shared gate / lambda gradients with the library's
all-reduce; the result must equal the gradients of the concatenated batch.
Timing reduction takes the slowest rank."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from sparse_rank_hybrid_simhash_b200 import distributed as DP
from sparse_rank_hybrid_simhash_b200.workloads import WORKLOADS, make_inputs

W = WORKLOADS["iid-4k"].replace(B=1, H=2, N=256, chunk=64, race_tables=4, race_bits=3)


def unit_grads(inp):
    """Sum of the shared-parameter gradients over the units of one batch."""
    gw = torch.zeros(2, W.d, dtype=torch.float64)
    gb = torch.zeros(2, dtype=torch.float64)
    gl = torch.zeros((), dtype=torch.float64)
    for b in range(W.B):
        for h in range(W.H):
            g = O.grads_head(inp["q"][b, h], inp["k"][b, h], inp["v"][b, h], inp["r_sort"],
                             inp["r_race"], W.chunk, inp["dy"][b, h], None, inp["gate_w"],
                             inp["gate_b"], float(inp["lam"][0]))
            gw += g["dgate_w"]
            gb += g["dgate_b"]
            gl += g["dlambda"]
    return gw, gb, gl.reshape(1)


def _rank(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        torch.set_num_threads(1)
        inp = make_inputs(W, seed=DP.rank_seed(W.seed, rank), with_dy=True)
        gw, gb, gl = unit_grads(inp)
        DP.allreduce_param_grads(gw, gb, gl)
        slowest = DP.max_over_ranks([float(rank + 1), 10.0 - rank], "cpu")
        out[rank] = (gw, gb, gl, slowest)
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_two_gloo_ranks_sum_shared_gradients():
    world = 2
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_rank, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    expect = [unit_grads(make_inputs(W, seed=DP.rank_seed(W.seed, r), with_dy=True))
              for r in range(world)]
    gw = expect[0][0] + expect[1][0]
    gb = expect[0][1] + expect[1][1]
    gl = expect[0][2] + expect[1][2]
    for r in range(world):
        rgw, rgb, rgl, slowest = out[r]
        assert torch.allclose(rgw, gw, atol=1e-12)
        assert torch.allclose(rgb, gb, atol=1e-12)
        assert torch.allclose(rgl, gl, atol=1e-12)
        assert slowest == [2.0, 10.0]


def test_rank_seeds_give_distinct_batches():
    a = make_inputs(W, seed=DP.rank_seed(W.seed, 0))
    b = make_inputs(W, seed=DP.rank_seed(W.seed, 1))
    assert not torch.equal(a["q"], b["q"])
