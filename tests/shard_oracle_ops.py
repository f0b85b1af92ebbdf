"""The fp64 oracle behind the device-step interface of the sequence sharding
(test infrastructure: lets the sharded scheme's routing, halo handling and
table sums run on the CPU, with gloo ranks, against the unsharded oracle)."""

from __future__ import annotations

import math

import torch

import oracle as O

F64 = torch.float64


def _units(x, B, H):
    return [x[b, h] for b in range(B) for h in range(H)]


def _order(p):
    return {0: "binary", 1: "gray", 2: "local"}[p.sort_order]


class OracleOps:
    """Same methods as shard.LibraryOps, computed by the oracle in fp64."""

    def sort_codes_of(self, p, q, k, r_sort, r_race):
        out = torch.empty((2, p.B, p.H, p.N), dtype=torch.int16)
        for i, (qu, ku) in enumerate(zip(_units(q, p.B, p.H), _units(k, p.B, p.H))):
            b, h = divmod(i, p.H)
            out[0, b, h] = O.simhash_codes(O.simhash_projections(qu, r_sort)).to(torch.int16)
            out[1, b, h] = O.simhash_codes(O.simhash_projections(ku, r_sort)).to(torch.int16)
        return out

    def sort_codes(self, p, code):
        perm = torch.empty((2, p.B, p.H, p.N), dtype=torch.int32)
        for w in range(2):
            for b in range(p.B):
                for h in range(p.H):
                    c = code[w, b, h].to(torch.int64) & 0xFFFF
                    perm[w, b, h] = O.stable_sort_perm(O.sort_keys(c, _order(p))).to(torch.int32)
        return perm

    def _rcodes(self, x, r_race):
        L, kr, d = r_race.shape
        return O.simhash_codes(O.simhash_projections(x, r_race.reshape(L * kr, d))
                               .reshape(x.shape[0], L, kr))

    def race_tables(self, p, k, v, r_race):
        NB = 1 << p.race_bits
        sums = torch.empty((p.B, p.H, p.race_tables, NB, p.d), dtype=F64)
        counts = torch.empty((p.B, p.H, p.race_tables, NB), dtype=torch.int32)
        for i, (ku, vu) in enumerate(zip(_units(k, p.B, p.H), _units(v, p.B, p.H))):
            b, h = divmod(i, p.H)
            c, s = O.race_build(self._rcodes(ku, r_race), vu.to(F64), NB)
            sums[b, h], counts[b, h] = s, c.to(torch.int32)
        return sums, counts

    def forward_tables(self, p, q, k, v, r_sort, r_race, gate_w, gate_b, lam, sums, counts):
        leaves = [t.detach().to(F64).requires_grad_(True) for t in (q, k, v, gate_w, gate_b)]
        lam64 = torch.tensor(float(lam.reshape(-1)[0]), dtype=F64, requires_grad=True)
        tab = sums.detach().to(F64).requires_grad_(True)
        qq, kk, vv, gw, gb = leaves
        scale = 1.0 / math.sqrt(p.d)
        ys = torch.empty(q.shape, dtype=F64)
        ys_list = []
        for i in range(p.B * p.H):
            b, h = divmod(i, p.H)
            qu, ku, vu = qq[b, h], kk[b, h], vv[b, h]
            with torch.no_grad():
                cq = O.simhash_codes(O.simhash_projections(qu, r_sort))
                ck = O.simhash_codes(O.simhash_projections(ku, r_sort))
                rq = self._rcodes(qu, r_race)
            pq = O.stable_sort_perm(O.sort_keys(cq, _order(p)))
            pk = O.stable_sort_perm(O.sort_keys(ck, _order(p)))
            o_sp, lse = O.sparse_branch(qu, ku, vu, pq, pk, p.chunk, scale, p.lookback)
            ctot, o_race, z_race = O.race_query(rq, counts[b, h].to(torch.int64), tab[b, h])
            if p.gate_fixed:
                g_s, g_r = O.gates(qu, None, None, fixed=(p.gate_s, p.gate_r))
            else:
                g_s, g_r = O.gates(qu, gw, gb)
            y, _ = O.fuse(o_sp, lse, o_race, z_race, g_s, g_r, lam64)
            ys_list.append(y)
        y = torch.stack(ys_list).view(q.shape)
        state = {"leaves": leaves + [lam64, tab], "y": y}
        return y.detach(), state

    def backward_tables(self, p, state, r_sort, r_race, gate_w, gate_b, lam, dy):
        loss = (state["y"] * dy.to(F64)).sum()
        g = torch.autograd.grad(loss, state["leaves"], allow_unused=True)
        zero = lambda t: torch.zeros_like(t)
        dq, dk, dv, dgw, dgb, dlam, dtab = [x if x is not None else zero(l)
                                            for x, l in zip(g, state["leaves"])]
        return dq, dk, dv, dgw, dgb, dlam.reshape(1), dtab

    def race_value_grad(self, p, k, r_race, d_sums, dv):
        for i, ku in enumerate(_units(k, p.B, p.H)):
            b, h = divmod(i, p.H)
            rk = self._rcodes(ku.to(F64), r_race)
            for l in range(p.race_tables):
                dv[b, h] += d_sums[b, h, l][rk[:, l]].to(dv.dtype)
