"""The host-batch pipeline (groups of heads streamed through the device)
against one whole-batch call of the same operator."""

import pytest
import torch

from sparse_rank_hybrid_simhash_b200 import binding as B
from sparse_rank_hybrid_simhash_b200.pipeline import HostStepPipeline
from sparse_rank_hybrid_simhash_b200.workloads import WORKLOADS, make_inputs, small

from parity import rel_l2

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("groups", [1, 2, 4])
def test_pipeline_matches_one_call(cuda_device, groups):
    w = small(WORKLOADS["text-32k"], B=2, H=2, N=1024)
    p = B.Params.from_workload(w)
    inp = make_inputs(w, with_dy=True)
    d = {k: t.to(cuda_device) for k, t in inp.items()}
    saved = B.alloc_saved(p, cuda_device)
    ws = B.alloc_workspace(p, cuda_device)
    y = B.forward(p, d["q"], d["k"], d["v"], d["r_sort"], d["r_race"], d["gate_w"], d["gate_b"],
                  d["lam"], saved=saved, ws=ws)
    ref = B.backward(p, d["q"], d["k"], d["v"], d["r_sort"], d["r_race"], d["gate_w"],
                     d["gate_b"], d["lam"], saved, d["dy"], ws=ws)
    torch.cuda.synchronize()
    host = {k: inp[k].pin_memory() for k in ("q", "k", "v", "dy")}
    outs = {k: torch.empty_like(host["q"], pin_memory=True) for k in ("y", "dq", "dk", "dv")}
    pipe = HostStepPipeline(p, groups, cuda_device, inp["r_sort"], inp["r_race"], inp["gate_w"],
                            inp["gate_b"], inp["lam"])
    for _ in range(2):   # a second step reuses both slots
        pipe.enqueue(host, outs)
        torch.cuda.synchronize()
        for name, want in (("y", y), ("dq", ref[0]), ("dk", ref[1]), ("dv", ref[2])):
            assert rel_l2(outs[name], want) <= 1e-3, name
        gw, gb, gl = pipe.gradients()
        for got, want in ((gw, ref[3]), (gb, ref[4]), (gl, ref[5])):
            assert rel_l2(got, want) <= 1e-4


def test_pipeline_chained_steps(cuda_device):
    """Back-to-back steps enqueued without a join between them (the next
    step's copy-in overlaps the last groups of the one before), each over its
    own host inputs and outputs, against one whole-batch call per step."""
    w = small(WORKLOADS["text-32k"], B=2, H=2, N=1024)
    p = B.Params.from_workload(w)
    base = make_inputs(w, with_dy=True)
    small_names = ("r_sort", "r_race", "gate_w", "gate_b", "lam")
    dsmall = {k: base[k].to(cuda_device) for k in small_names}
    pipe = HostStepPipeline(p, 4, cuda_device, *(base[k] for k in small_names))
    steps = []
    for seed in (11, 12, 13):
        inp = make_inputs(w, seed=seed, with_dy=True)
        host = {k: inp[k].pin_memory() for k in ("q", "k", "v", "dy")}
        outs = {k: torch.empty_like(host["q"], pin_memory=True) for k in ("y", "dq", "dk", "dv")}
        steps.append((inp, host, outs))
    for _, host, outs in steps:
        pipe.enqueue_chained(host, outs)
    pipe.join()
    torch.cuda.synchronize()
    saved = B.alloc_saved(p, cuda_device)
    ws = B.alloc_workspace(p, cuda_device)
    for inp, _, outs in steps:
        d = {k: inp[k].to(cuda_device) for k in ("q", "k", "v", "dy")}
        y = B.forward(p, d["q"], d["k"], d["v"], *(dsmall[k] for k in small_names),
                      saved=saved, ws=ws)
        ref = B.backward(p, d["q"], d["k"], d["v"], *(dsmall[k] for k in small_names), saved,
                         d["dy"], ws=ws)
        torch.cuda.synchronize()
        for name, want in (("y", y), ("dq", ref[0]), ("dk", ref[1]), ("dv", ref[2])):
            assert rel_l2(outs[name], want) <= 1e-3, name
    # the parameter-gradient partial sums are those of the last step
    gw, gb, gl = pipe.gradients()
    for got, want in ((gw, ref[3]), (gb, ref[4]), (gl, ref[5])):
        assert rel_l2(got, want) <= 1e-4
