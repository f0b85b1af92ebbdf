"""Sequence sharding with the library's kernels on one GPU: every rank of the
group in one process (LocalComm: the collectives are device copies), against
the fp64 oracle on the whole sequence and against one unsharded call."""

import pytest
import torch

from sparse_rank_hybrid_simhash_b200 import binding as B
from sparse_rank_hybrid_simhash_b200.shard import LocalComm, ShardedElsaa
from sparse_rank_hybrid_simhash_b200.workloads import WORKLOADS, make_inputs, small

from parity import assert_close, check_param_grads, oracle_unit, rel_l2

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,N,P", [("text-32k", 2048, 2), ("text-32k", 2048, 4),
                                      ("iid-4k", 1024, 2)])
def test_sharded_sequence_matches_oracle(cuda_device, name, N, P):
    w = small(WORKLOADS[name], B=1, H=2, N=N)
    p = B.Params.from_workload(w)
    inp = make_inputs(w, with_dy=True)
    d = {k: t.to(cuda_device) for k, t in inp.items()}
    M = N // P
    sh = {n: [d[n][:, :, r * M:(r + 1) * M].contiguous() for r in range(P)]
          for n in ("q", "k", "v", "dy")}
    s = ShardedElsaa(p, LocalComm(P))
    args = (d["r_sort"], d["r_race"], d["gate_w"], d["gate_b"], d["lam"])
    ys = s.forward(sh["q"], sh["k"], sh["v"], *args)
    grads, shared = s.backward(sh["dy"], *args)
    torch.cuda.synchronize()
    y = torch.cat(ys, dim=2).cpu()
    dq, dk, dv = (torch.cat([g[j] for g in grads], dim=2).cpu() for j in range(3))
    # against the oracle, unit by unit on the whole sequence, and the shared
    # gradients (summed over ranks) against the oracle's sums
    refs = []
    for b in range(w.B):
        for h in range(w.H):
            ref = oracle_unit(w, inp, b, h, backward=True)
            refs.append(ref)
            assert_close("y", y[b, h], ref["y"], w.dtype)
            assert_close("dq", dq[b, h], ref["grad_dq"], w.dtype)
            assert_close("dk", dk[b, h], ref["grad_dk"], w.dtype)
            assert_close("dv", dv[b, h], ref["grad_dv"], w.dtype)
    check_param_grads(w, {"dgate_w": shared[0].cpu(), "dgate_b": shared[1].cpu(),
                          "dlambda": shared[2].cpu()}, refs)
    # against one unsharded call of the same operator
    saved = B.alloc_saved(p, cuda_device)
    ws = B.alloc_workspace(p, cuda_device)
    y1 = B.forward(p, d["q"], d["k"], d["v"], *args, saved=saved, ws=ws)
    g1 = B.backward(p, d["q"], d["k"], d["v"], d["r_sort"], d["r_race"], d["gate_w"],
                    d["gate_b"], d["lam"], saved, d["dy"], ws=ws)
    torch.cuda.synchronize()
    # the same kernels on other row groupings: within bf16 rounding of each other
    assert rel_l2(y, y1) <= 2e-3
    for got, want in zip((dq, dk, dv), g1[:3]):
        assert rel_l2(got, want) <= 2e-3
