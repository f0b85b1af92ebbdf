"""A sequence split across devices: the ELSAA operator over token shards.

For sequences too long for one device ("Two Efficient Attentions, One
Denominator Problem", section "Length extrapolation is the strongest
robustness signal": needle retrieval at extreme lengths), every (batch, head)
unit's N tokens are split into P contiguous shards of M = N / P tokens, one per
rank.  The operator's structure makes the split exact:

  * Sort-LSH orders Q and K by hash code over the whole sequence.  Every
    rank's sort codes are gathered, so every rank computes the same global
    orders (stable, ties by token index) and knows where each row goes.
  * Rank r takes the queries of sorted ranks [r M, (r + 1) M) and the keys of
    sorted ranks [r M - H, (r + 1) M), H = lookback * chunk (the chunks the
    first query chunk looks back on), in sorted order; H zero query rows pad
    the front.  The library's own stable sort of these rows is the identity,
    so its chunks are the global chunks and its sparse branch is the global
    one for the rank's queries.  (M must be a multiple of the chunk, M >= H.)
  * RACE tables are sums over keys: every rank builds its shard's tables and
    one all-reduce gives the whole sequence's tables, which the rank's forward
    reads.  In the backward the table gradient is summed the same way and the
    RACE value gradient is gathered on the key's own shard.
  * Outputs and gradients go back to the token's shard; a key's sparse
    gradient gets contributions from the rank holding its sorted position and
    from the next rank's front chunks, and they are added there.

The exchanges are all-to-all collectives (torch.distributed: NCCL on GPUs,
gloo on the CPU); the device work is the library's (ops.LibraryOps), or any
object with the same methods.  One hash round, non-causal (a causal mask needs
token indices the local problem does not see).

The code is written for a list of ranks driven by this process: one rank per
process under torch.distributed (DistComm), or every rank of the group in one
process (LocalComm, which emulates the collectives by local copies).
"""

from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import torch

from . import binding as Bn


# ---------------------------------------------------------------------------
# collectives over the ranks this process drives
# ---------------------------------------------------------------------------

class LocalComm:
    """Every rank of the group in this process: collectives are local copies."""

    def __init__(self, world: int):
        self.world = world
        self.ranks = list(range(world))

    def all_gather(self, xs: List[torch.Tensor]) -> List[List[torch.Tensor]]:
        return [[x.clone() for x in xs] for _ in xs]

    def all_reduce_(self, xs: List[torch.Tensor]) -> None:
        tot = xs[0].clone()
        for x in xs[1:]:
            tot += x
        for x in xs:
            x.copy_(tot)

    def all_to_all(self, sends: List[List[torch.Tensor]]) -> List[List[torch.Tensor]]:
        """sends[i][d]: rows rank i sends to rank d; returns recv[i][s]."""
        return [[sends[s][d] for s in range(self.world)] for d in range(self.world)]


class DistComm:
    """One rank per process (torch.distributed, any backend)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.ranks = [dist.get_rank(group)]

    def all_gather(self, xs: List[torch.Tensor]) -> List[List[torch.Tensor]]:
        out = [torch.empty_like(xs[0]) for _ in range(self.world)]
        self.dist.all_gather(out, xs[0].contiguous(), group=self.group)
        return [out]

    def all_reduce_(self, xs: List[torch.Tensor]) -> None:
        self.dist.all_reduce(xs[0], group=self.group)

    def all_to_all(self, sends: List[List[torch.Tensor]]) -> List[List[torch.Tensor]]:
        send = sends[0]
        width = send[0].shape[1:]
        counts = torch.tensor([t.shape[0] for t in send], dtype=torch.int64)
        if send[0].is_cuda:
            counts = counts.cuda()
        rc = torch.empty_like(counts)
        self.dist.all_to_all_single(rc, counts, group=self.group)
        rc = rc.tolist()
        flat = torch.cat([t.reshape(t.shape[0], -1) for t in send])
        recv = torch.empty((sum(rc), flat.shape[1]), dtype=flat.dtype, device=flat.device)
        self.dist.all_to_all_single(recv, flat, output_split_sizes=rc,
                                    input_split_sizes=[t.shape[0] for t in send], group=self.group)
        return [[x.view(-1, *width) for x in recv.split(rc)]]


# ---------------------------------------------------------------------------
# routes: which rows go where
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class Routes:
    """For one rank: rows it sends to every rank (indices into its flat shard
    [BH * M]) and where the rows it receives from every rank go (indices into
    its flat local problem [BH * N_loc]), in matching order."""
    send: List[torch.Tensor]
    recv: List[torch.Tensor]


def front(r: int, halo: int) -> int:
    """Rows in front of rank r's own sorted range: the look-back chunks (none for rank 0)."""
    return halo if r > 0 else 0


def routes(perm: torch.Tensor, r: int, world: int, M: int, halo: int, with_front: bool) -> Routes:
    """perm [BH, N]: token index at each global sorted rank (one of Q or K).
    Destination d's local rows i in [0, M + front) hold sorted ranks
    d M - front + i; with_front = False leaves the front rows empty (queries)."""
    BH, N = perm.shape
    dev = perm.device
    send, recv = [], []
    for d in range(world):
        f = front(d, halo)
        lo = d * M - (f if with_front else 0)
        tok = perm[:, lo:(d + 1) * M]                        # [BH, rows]
        i = torch.arange(tok.shape[1], device=dev) + (0 if with_front else f)
        src = torch.div(tok, M, rounding_mode="floor")
        unit = torch.arange(BH, device=dev)[:, None].expand_as(tok)
        m = src == r
        send.append((unit * M + (tok - r * M))[m].to(torch.int64))
        if d == r:
            nloc = M + f
            recv = [((unit * nloc + i[None, :])[src == s]).to(torch.int64) for s in range(world)]
    return Routes(send, recv)


def exchange(comm, routes_all: List[Routes], xs: List[torch.Tensor],
             out_rows: List[int], fill=0.0) -> List[torch.Tensor]:
    """Rows of each rank's flat shard xs[i] [BH * M, ...] to the local problems:
    returns, per rank, a zero-filled [out_rows[i], ...] with the received rows
    placed at their routes."""
    sends = [[x.index_select(0, idx) for idx in rt.send] for x, rt in zip(xs, routes_all)]
    recvs = comm.all_to_all(sends)
    outs = []
    for i, (rt, rv) in enumerate(zip(routes_all, recvs)):
        o = torch.full((out_rows[i],) + tuple(xs[i].shape[1:]), fill, dtype=xs[i].dtype,
                       device=xs[i].device)
        for s, rows in enumerate(rv):
            if rows.shape[0]:
                o.index_copy_(0, rt.recv[s], rows)
        outs.append(o)
    return outs


def exchange_back(comm, routes_all: List[Routes], ys: List[torch.Tensor], shard_rows: int,
                  add: bool, acc_dtype=None) -> List[torch.Tensor]:
    """The reverse: rows of each rank's local problem ys[i] [BH * N_loc, ...]
    back to the ranks holding their tokens; add = True sums rows that arrive
    from several ranks (key gradients), in acc_dtype."""
    sends = [[y.index_select(0, idx) for idx in rt.recv] for y, rt in zip(ys, routes_all)]
    recvs = comm.all_to_all(sends)
    outs = []
    for i, (rt, rv) in enumerate(zip(routes_all, recvs)):
        dt = acc_dtype or ys[i].dtype
        o = torch.zeros((shard_rows,) + tuple(ys[i].shape[1:]), dtype=dt, device=ys[i].device)
        for d, rows in enumerate(rv):
            if rows.shape[0]:
                if add:
                    o.index_add_(0, rt.send[d], rows.to(dt))
                else:
                    o.index_copy_(0, rt.send[d], rows.to(dt))
        outs.append(o)
    return outs


# ---------------------------------------------------------------------------
# the library as the device steps
# ---------------------------------------------------------------------------

class LibraryOps:
    """Device steps of the sharded operator: the libelsaa entry points."""

    def sort_codes_of(self, p, q, k, r_sort, r_race):
        return Bn.sort_codes_of(p, q, k, r_sort, r_race)

    def sort_codes(self, p, code):
        return Bn.sort_codes(p, code)

    def race_tables(self, p, k, v, r_race):
        return Bn.race_tables(p, k, v, r_race)

    def forward_tables(self, p, q, k, v, r_sort, r_race, gate_w, gate_b, lam, sums, counts):
        saved = Bn.alloc_saved(p, q.device)
        ws = Bn.alloc_workspace(p, q.device)
        y = Bn.forward_tables(p, q, k, v, r_sort, r_race, gate_w, gate_b, lam, sums, counts,
                              saved=saved, ws=ws)
        return y, {"saved": saved, "ws": ws, "q": q, "k": k, "v": v}

    def backward_tables(self, p, state, r_sort, r_race, gate_w, gate_b, lam, dy):
        return Bn.backward_tables(p, state["q"], state["k"], state["v"], r_sort, r_race, gate_w,
                                  gate_b, lam, state["saved"], dy, ws=state["ws"])

    def race_value_grad(self, p, k, r_race, d_sums, dv):
        Bn.race_value_grad(p, k, r_race, d_sums, dv)


# ---------------------------------------------------------------------------
# the sharded operator
# ---------------------------------------------------------------------------

def shard_params(p: Bn.Params, N: int) -> Bn.Params:
    """The same problem with N tokens per unit."""
    q = Bn.Params.from_buffer_copy(bytes(p))
    q.N = N
    return q


class ShardedElsaa:
    """Forward and backward of ELSAA over P token shards.

    p: the whole sequence's parameters (N = P M).  comm: LocalComm (all ranks
    here) or DistComm (this process's rank).  Inputs per driven rank: q, k, v
    (and dy) [B, H, M, d] shards; the hyperplanes, gate weights and lambda
    are the same on every rank."""

    def __init__(self, p: Bn.Params, comm, ops=None):
        self.p = p
        self.comm = comm
        self.ops = ops or LibraryOps()
        P = comm.world
        if p.N % P:
            raise ValueError("N must be a multiple of the number of shards")
        self.M = p.N // P
        self.halo = p.lookback * p.chunk
        if self.M % p.chunk or self.M < self.halo:
            raise ValueError("the shard length must be a multiple of the chunk and cover the "
                             "look-back chunks")
        if p.hash_rounds > 1 or p.causal:
            raise ValueError("sharding takes one hash round and no causal mask")
        self.p_shard = shard_params(p, self.M)

    def forward(self, q: List[torch.Tensor], k: List[torch.Tensor], v: List[torch.Tensor],
                r_sort, r_race, gate_w, gate_b, lam) -> List[torch.Tensor]:
        p, ops, comm, M, H = self.p, self.ops, self.comm, self.M, self.halo
        B, Hh, d = p.B, p.H, p.d
        BH = B * Hh
        ranks = comm.ranks
        # 1. sort codes of every shard, gathered: every rank orders the whole sequence
        # (codes travel as int32: collectives have no 16-bit integer type)
        codes = [ops.sort_codes_of(self.p_shard, qi, ki, r_sort, r_race).to(torch.int32)
                 for qi, ki in zip(q, k)]
        gathered = comm.all_gather(codes)                     # per rank: [P] x [2, B, H, M]
        perms = []
        for g in gathered:
            full = torch.cat(g, dim=-1).to(torch.int16).contiguous()   # [2, B, H, N] token order
            perms.append(ops.sort_codes(p, full).view(2, BH, p.N).to(torch.int64))
        # 2. RACE tables of every shard, summed
        tabs = [ops.race_tables(self.p_shard, ki, vi, r_race) for ki, vi in zip(k, v)]
        comm.all_reduce_([t[0] for t in tabs])
        comm.all_reduce_([t[1] for t in tabs])
        # 3. rows of each rank's sorted range (keys with the front chunks)
        self.rq = [routes(pm[0], r, comm.world, M, H, False) for pm, r in zip(perms, ranks)]
        self.rk = [routes(pm[1], r, comm.world, M, H, True) for pm, r in zip(perms, ranks)]
        nloc = [M + front(r, H) for r in ranks]
        rows = [BH * n for n in nloc]
        flat = lambda ts: [t.reshape(BH * M, d) for t in ts]
        ql = exchange(comm, self.rq, flat(q), rows)
        kl = exchange(comm, self.rk, flat(k), rows)
        vl = exchange(comm, self.rk, flat(v), rows)
        # 4. each rank's problem with the summed tables
        self.local = []
        ys = []
        for i, r in enumerate(ranks):
            pl = shard_params(p, nloc[i])
            shape = (B, Hh, nloc[i], d)
            y, st = ops.forward_tables(pl, ql[i].view(shape), kl[i].view(shape),
                                       vl[i].view(shape), r_sort, r_race, gate_w, gate_b, lam,
                                       tabs[i][0], tabs[i][1])
            self.local.append((pl, st))
            ys.append(y.reshape(BH * nloc[i], d))
        self.k_shards = k
        self.rows = rows
        out = exchange_back(comm, self.rq, ys, BH * M, add=False)
        return [o.view(B, Hh, M, d) for o in out]

    def backward(self, dy: List[torch.Tensor], r_sort, r_race, gate_w, gate_b, lam):
        """Gradients of sum(y dy): per rank (dq, dk, dv) shards and the shared
        (dgate_w, dgate_b, dlambda), summed over every rank."""
        p, ops, comm, M = self.p, self.ops, self.comm, self.M
        B, Hh, d = p.B, p.H, p.d
        BH = B * Hh
        dyl = exchange(comm, self.rq, [t.reshape(BH * M, d) for t in dy], self.rows)
        res = []
        for i, (pl, st) in enumerate(self.local):
            shape = (B, Hh, pl.N, d)
            res.append(ops.backward_tables(pl, st, r_sort, r_race, gate_w, gate_b, lam,
                                           dyl[i].view(shape)))
        # shared gradients and the table gradient, summed over every rank
        comm.all_reduce_([x[6] for x in res])
        for j in (3, 4, 5):
            comm.all_reduce_([x[j] for x in res])
        flat_loc = lambda j: [x[j].reshape(-1, d) for x in res]
        dq = exchange_back(comm, self.rq, flat_loc(0), BH * M, add=False)
        acc = torch.promote_types(dy[0].dtype, torch.float32)   # at least fp32 for the sums
        dk = exchange_back(comm, self.rk, flat_loc(1), BH * M, add=True, acc_dtype=acc)
        dv = exchange_back(comm, self.rk, flat_loc(2), BH * M, add=True, acc_dtype=acc)
        dt = dy[0].dtype
        out = []
        for i in range(len(res)):
            dvi = dv[i].to(dt).view(B, Hh, M, d).contiguous()
            # the RACE branch's value gradient, on the key's own shard
            ops.race_value_grad(self.p_shard, self.k_shards[i], r_race, res[i][6], dvi)
            out.append((dq[i].view(B, Hh, M, d), dk[i].to(dt).view(B, Hh, M, d), dvi))
        dgw, dgb, dlam = res[0][3], res[0][4], res[0][5]
        return out, (dgw, dgb, dlam)
