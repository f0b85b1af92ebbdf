"""Sequence sharding (shard.py) on the CPU: the sharded scheme's routing,
front chunks and summed RACE tables, with the oracle as the device steps,
against the unsharded oracle.  Every rank in one process (LocalComm) and two
gloo ranks (DistComm)."""

import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from sparse_rank_hybrid_simhash_b200 import binding as B
from sparse_rank_hybrid_simhash_b200.shard import DistComm, LocalComm, ShardedElsaa, routes

from shard_oracle_ops import OracleOps

F64 = torch.float64


def problem(N=256, d=8, chunk=16, lookback=1, order="binary", seed=0):
    g = torch.Generator().manual_seed(seed)
    Bb, H, bs, L, kr = 1, 2, 3, 3, 3
    p = B.Params.make(Bb, H, N, d, "f32", bs, chunk, L, kr, sort_order=order, lookback=lookback)
    t = {n: torch.randn(Bb, H, N, d, generator=g, dtype=F64) for n in ("q", "k", "v", "dy")}
    t["r_sort"] = torch.randn(bs, d, generator=g, dtype=F64)
    t["r_race"] = torch.randn(L, kr, d, generator=g, dtype=F64)
    t["gate_w"] = 0.3 * torch.randn(2, d, generator=g, dtype=F64)
    t["gate_b"] = torch.randn(2, generator=g, dtype=F64)
    t["lam"] = torch.tensor([0.8], dtype=F64)
    return p, t


def reference(p, t):
    out = {n: torch.empty_like(t["q"]) for n in ("y", "dq", "dk", "dv")}
    dgw = torch.zeros(2, p.d, dtype=F64)
    dgb = torch.zeros(2, dtype=F64)
    dlam = torch.zeros((), dtype=F64)
    order = {0: "binary", 1: "gray", 2: "local"}[p.sort_order]
    for b in range(p.B):
        for h in range(p.H):
            g = O.grads_head(t["q"][b, h], t["k"][b, h], t["v"][b, h], t["r_sort"], t["r_race"],
                             p.chunk, t["dy"][b, h], None, t["gate_w"], t["gate_b"],
                             float(t["lam"][0]), sort_order=order, lookback=p.lookback)
            out["y"][b, h], out["dq"][b, h], out["dk"][b, h], out["dv"][b, h] = \
                g["y"], g["dq"], g["dk"], g["dv"]
            dgw += g["dgate_w"]
            dgb += g["dgate_b"]
            dlam += g["dlambda"]
    return out, (dgw, dgb, dlam)


def shards(t, P, ranks):
    M = t["q"].shape[2] // P
    return {n: [t[n][:, :, r * M:(r + 1) * M].contiguous() for r in ranks]
            for n in ("q", "k", "v", "dy")}


def run_sharded(p, t, comm):
    sh = shards(t, comm.world, comm.ranks)
    s = ShardedElsaa(p, comm, OracleOps())
    args = (t["r_sort"], t["r_race"], t["gate_w"], t["gate_b"], t["lam"])
    ys = s.forward(sh["q"], sh["k"], sh["v"], *args)
    grads, shared = s.backward(sh["dy"], *args)
    return ys, grads, shared


def check(p, t, comm, ys, grads, shared, ref, ref_shared):
    M = p.N // comm.world
    for i, r in enumerate(comm.ranks):
        sl = slice(r * M, (r + 1) * M)
        assert torch.allclose(ys[i], ref["y"][:, :, sl], atol=1e-10), f"y rank {r}"
        for j, n in enumerate(("dq", "dk", "dv")):
            assert torch.allclose(grads[i][j], ref[n][:, :, sl], atol=1e-10), f"{n} rank {r}"
    for got, want in zip(shared, ref_shared):
        assert torch.allclose(got.reshape(-1), want.reshape(-1), atol=1e-10)


@pytest.mark.parametrize("P,lookback,order", [(2, 1, "binary"), (4, 1, "binary"),
                                              (2, 2, "gray"), (4, 1, "local")])
def test_sharded_equals_unsharded(P, lookback, order):
    p, t = problem(lookback=lookback, order=order)
    ref, ref_shared = reference(p, t)
    comm = LocalComm(P)
    ys, grads, shared = run_sharded(p, t, comm)
    check(p, t, comm, ys, grads, shared, ref, ref_shared)


def test_routes_place_every_row_once():
    # every sorted query rank lands in exactly one rank's range, every key rank
    # in its own range and (the last look-back chunks) in the next rank's front
    g = torch.Generator().manual_seed(3)
    BH, N, P, halo = 3, 96, 3, 16
    M = N // P
    perm = torch.stack([torch.randperm(N, generator=g) for _ in range(BH)])
    for with_front in (False, True):
        got = torch.zeros(BH, N, dtype=torch.int64)
        for r in range(P):
            rt = routes(perm, r, P, M, halo, with_front)
            for d in range(P):
                got.view(-1).index_add_(0, (rt.send[d] // M) * N + r * M + rt.send[d] % M,
                                        torch.ones_like(rt.send[d]))
        expect = torch.ones(BH, N, dtype=torch.int64)
        if with_front:
            ranks = torch.empty_like(perm)
            ranks.scatter_(1, perm, torch.arange(N).expand(BH, N))
            expect += ((ranks % M >= M - halo) & (ranks < N - M)).to(torch.int64)
        assert torch.equal(got, expect)


def test_invalid_shardings_are_rejected():
    p, _ = problem(N=256, chunk=16)
    with pytest.raises(ValueError):
        ShardedElsaa(p, LocalComm(3))            # 256 tokens do not split in 3
    p2, _ = problem(N=256, chunk=64, lookback=1)
    with pytest.raises(ValueError):
        ShardedElsaa(p2, LocalComm(8))           # 32-token shards, 64-token chunks
    p3, _ = problem()
    p3.hash_rounds = 2
    with pytest.raises(ValueError):
        ShardedElsaa(p3, LocalComm(2))


def _gloo_rank(rank, world, port, result_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        p, t = problem(seed=5)
        ref, ref_shared = reference(p, t)
        comm = DistComm()
        ys, grads, shared = run_sharded(p, t, comm)
        check(p, t, comm, ys, grads, shared, ref, ref_shared)
        open(os.path.join(result_dir, f"ok{rank}"), "w").close()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    port = 29500 + (os.getpid() % 1000)
    mp.start_processes(_gloo_rank, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    assert os.path.exists(tmp_path / "ok0") and os.path.exists(tmp_path / "ok1")
