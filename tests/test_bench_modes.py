"""Host logic of the bench's ablation / single-branch modes (no GPU): each
mode sets the gates and lambda of the method's ablations, and the oracle under
those settings reduces to the branch the mode names."""

import importlib.util
import os

import pytest
import torch

import oracle as O
from sparse_rank_hybrid_simhash_b200.workloads import WORKLOADS, make_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_mode_settings():
    bench = _bench()
    w = WORKLOADS["text-32k"]
    assert bench.apply_mode(w, "elsaa") == w
    s = bench.apply_mode(w, "sort_lsh_race")
    assert (s.gate_fixed, s.lam) == (False, 0.0)
    r = bench.apply_mode(w, "race_only")
    assert (r.gate_fixed, r.gate_s, r.gate_r, r.lam) == (True, 0.0, 1.0, w.lam)
    p = bench.apply_mode(w, "sparse_only")
    assert (p.gate_fixed, p.gate_s, p.gate_r, p.lam) == (True, 1.0, 0.0, 0.0)
    cfg = bench.bench_config(p, "sparse_only", 1, "x")
    assert cfg["mode"] == "sparse_only" and cfg["gates"] == "fixed 1.0/0.0" and cfg["lambda"] == 0.0


@pytest.mark.parametrize("mode,branch", [("race_only", "o_race"), ("sparse_only", "o_sp")])
def test_single_branch_modes_reduce_to_their_branch(mode, branch):
    bench = _bench()
    w = bench.apply_mode(WORKLOADS["iid-4k"].replace(B=1, H=1, N=256, chunk=64), mode)
    inp = make_inputs(w, with_dy=False)
    gw = None if w.gate_fixed else inp["gate_w"][0]
    ref = O.forward_head(inp["q"][0, 0], inp["k"][0, 0], inp["v"][0, 0], inp["r_sort"],
                         inp["r_race"], w.chunk, gate_w=gw, gate_b=inp["gate_b"],
                         fixed_gates=(w.gate_s, w.gate_r) if w.gate_fixed else None,
                         lam=float(inp["lam"][0]))
    assert torch.allclose(ref["y"], ref[branch], rtol=0, atol=1e-12)


def test_operator_roofline_of_the_text_workload():
    # the operator roofline the bench divides by: fwd 1.04e11 flops / 0.403 GB,
    # fwd+bwd 2.33e11 flops / 1.32 GB at B2 H12 N32768 d64 bf16, c 128, 7 + 32 x 8 bits
    bench = _bench()
    peaks = {"bf16_tflops": 1606.3, "hbm_gbs": 6539.5}
    r = bench.operator_roofline(WORKLOADS["text-32k"], peaks)
    n, bh, d = 32768, 24, 64
    window = 128 * (128 + 255 * 256)          # chunk 0 sees 128 keys, the rest 256
    assert bench.window_keys(n, 128) == window
    f_fwd = 2 * 2 * bh * n * d * (7 + 32 * 8) + 4 * bh * window * d
    assert abs(r["flops_fwd"] - f_fwd) < 1
    assert abs(r["bytes_fwd"] - 4 * bh * n * d * 2) < 1
    assert abs(r["fwd_us"] - 65.0) < 0.1 and abs(r["fwdbwd_us"] - 202.0) < 0.1
    # lookback widens the window: chunk j sees min(j, lb) + 1 chunks
    assert bench.window_keys(1024, 128, 3) == 128 * 128 * sum(min(j, 3) + 1 for j in range(8))


def test_recorded_traffic_only_describes_the_captured_kernels(monkeypatch):
    # DRAM bytes from a capture at 12 heads scale with the units of the run and
    # are withheld where the run launches something else or the kernel's
    # source has changed since the capture
    import hashlib
    bench = _bench()
    src = "sparse_rank_hybrid_simhash_b200/csrc/attn_tc_bwd3.cu"
    sha = hashlib.sha1(open(os.path.join(ROOT, src), "rb").read()).hexdigest()
    monkeypatch.setitem(bench.RECORDED_TRAFFIC, "sparse_bwd", (src, sha, 3.0e8, "tc_attn"))
    monkeypatch.setitem(bench.RECORDED_TRAFFIC, "race_fuse", (src, sha, 1.0e8, "slab_fwd"))
    w = WORKLOADS["text-32k"]
    path = {"tc_hash": True, "tc_attn": True, "slab_fwd": True, "slab_bwd": True}
    assert bench.recorded_traffic(w, "sparse_bwd", path) == 3.0e8 * 24 / 12
    assert bench.recorded_traffic(w.replace(B=1), "sparse_bwd", path) == 3.0e8
    assert bench.recorded_traffic(w, "race_fuse", dict(path, slab_fwd=False)) is None
    assert bench.recorded_traffic(w.replace(lookback=2), "sparse_bwd", path) is None
    assert bench.recorded_traffic(WORKLOADS["iid-4k"], "sparse_bwd", path) is None
    assert bench.recorded_traffic(bench.apply_mode(w, "race_only"), "sparse_bwd", path) is None
    monkeypatch.setitem(bench.RECORDED_TRAFFIC, "sparse_bwd", (src, "0" * 40, 3.0e8, "tc_attn"))
    assert bench.recorded_traffic(w, "sparse_bwd", path) is None
