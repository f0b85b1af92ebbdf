"""Full-size GPU parity: the workloads at their real sizes, in the launch
configuration the benchmark times.  The oracle recomputes sampled (batch,
head) units one by one (units are independent); properties that hold for
every unit are checked on all of them."""

import pytest
import torch

import oracle as O
from sparse_rank_hybrid_simhash_b200 import binding as B
from sparse_rank_hybrid_simhash_b200.workloads import WORKLOADS, make_inputs

from parity import assert_close, check_param_grads, check_unit, run_gpu

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _invariants(w, views):
    """Every unit: permutations are permutations, codes are nondecreasing
    along them with increasing token index on ties, every table's counts sum
    to N, and Ctot equals the sum of the query's bucket counts."""
    BH, N, L = w.B * w.H, w.N, w.race_tables
    dev = "cuda"
    for which in ("q", "k"):
        perm = views["perm_" + which].to(dev).reshape(BH, N).long()
        code = (views["code_" + which].to(dev).reshape(BH, N).long() & 0xFFFF)
        assert torch.equal(perm.sort(dim=1).values,
                           torch.arange(N, device=dev).expand(BH, N)), which
        c = code.gather(1, perm)
        assert bool((c[:, 1:] >= c[:, :-1]).all()), which
        ties = c[:, 1:] == c[:, :-1]
        assert bool((perm[:, 1:] > perm[:, :-1])[ties].all()), which
    counts = views["race_count"].to(dev).reshape(BH, L, -1).long()
    assert bool((counts.sum(-1) == N).all())
    rq = views["rcode_q"].to(dev).reshape(BH, N, L).long() & 0xFFFF
    expect = counts.gather(2, rq.permute(0, 2, 1)).sum(1)       # [BH, N]
    assert torch.equal(views["ctot"].to(dev).reshape(BH, N).long(), expect)


@pytest.mark.parametrize("name,units", [
    ("text-32k", [(0, 0), (1, 11)]),
    ("vision-16k", [(0, 3), (7, 7)]),
])
def test_full_size_forward_backward_sampled_units(cuda_device, name, units):
    w = WORKLOADS[name]
    inp = make_inputs(w, with_dy=True)
    gpu = run_gpu(w, inp, backward=True)
    _invariants(w, gpu["views"])
    report = {}
    for (b, h) in units:
        check_unit(w, inp, gpu, b, h, True, report)
    codes = w.B * w.H * w.N * (w.race_tables + 1) * 2
    assert report.get("code_mismatch_near_zero", 0) <= 1e-4 * codes


def test_full_size_iid_4k_every_unit_and_parameter_gradients(cuda_device):
    w = WORKLOADS["iid-4k"]
    inp = make_inputs(w, with_dy=True)
    gpu = run_gpu(w, inp, backward=True)
    _invariants(w, gpu["views"])
    report = {}
    refs = [check_unit(w, inp, gpu, b, h, True, report) for b in range(w.B) for h in range(w.H)]
    check_param_grads(w, gpu, refs)


def test_full_size_needle_forward_and_needle_weight(cuda_device):
    w = WORKLOADS["needle-256k"]
    inp = make_inputs(w, with_dy=False)
    gpu = run_gpu(w, inp, backward=False)
    _invariants(w, gpu["views"])
    b, h = 0, 5
    check_unit(w, inp, gpu, b, h, False, {})
    # the needle row's total output weight on the planted value: a second
    # forward with V = 0 except v_p = 1 puts that weight in every coordinate
    p = int(inp["needle_key"][b, h])
    c = int(inp["needle_query"][b, h])
    v1 = torch.zeros_like(inp["v"])
    v1[b, h, p] = 1.0
    inp1 = dict(inp, v=v1)
    gpu1 = run_gpu(w, inp1, backward=False)
    ref1 = O.forward_head(inp1["q"][b, h], inp1["k"][b, h], inp1["v"][b, h], inp1["r_sort"],
                          inp1["r_race"], w.chunk, None, inp1["gate_w"], inp1["gate_b"],
                          float(inp1["lam"][0]))
    got = gpu1["y"][b, h, c].double()
    assert_close("needle weight", got, ref1["y"][c], "bf16")
    # planted key = 4 x the chosen query: same sort code and every RACE code
    assert int(ref1["code_q"][c]) == int(ref1["code_k"][p])
    assert torch.equal(ref1["rcode_q"][c], ref1["rcode_k"][p])
