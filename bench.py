"""Benchmark of the ELSAA attention operator (libelsaa) on B200.

One step = one forward and one backward of the whole operator (SimHash codes,
Sort-LSH order, RACE build, sparse branch, RACE gather + fusion, and their
backward) over one batch of the text-32k workload: B2 H12 N32768 d64 bf16,
7-bit Sort-LSH, chunk 128, RACE 32 x 8-bit, learned gates.  Inputs are seeded
synthetic tensors resident in HBM before the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--mode elsaa|sort_lsh_race|race_only|sparse_only]
                    [--sort-order binary|gray|local] [--lookback L] [--hash-rounds R]
                    [--causal]
                    [--dense-context] [--no-cpu-baseline] [--no-other-workloads]
                    [--seq-shards P]

The modes are the method's ablations on the same kernels (lambda = 0, or one
branch gated off); sort order, lookback and causal select the extensions of
the Sort-LSH window; --dense-context adds a timing of dense torch SDPA on the
same inputs as context.

Multi-GPU (torchrun, one rank per GPU): every rank runs its own batch (weak
scaling, different seed per rank); the shared gate and lambda gradients are
summed across ranks with one NCCL all-reduce inside the step.  Time is device
time (CUDA events on the launching stream), max over ranks.  Rank 0 prints one
JSON line.

``--seq-shards P`` times instead the workload with every unit's sequence split
into P token shards (shard.py): one per rank under torchrun, or all of them in
one process on one GPU (an emulation; the line says so).

``--impl reference`` times the fp64 CPU oracle (the reference arm: there is no
runnable reference implementation) on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from sparse_rank_hybrid_simhash_b200 import binding as B  # noqa: E402
from sparse_rank_hybrid_simhash_b200 import distributed as DP  # noqa: E402
from sparse_rank_hybrid_simhash_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

METRIC = "ELSAA attn tokens/s fwd and fwd+bwd at N=32K,d=64 bf16; % of roofline"
WORKLOAD = "text-32k"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "sm_max_mhz": p.get("sm_max_mhz", 1965.0), "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "sm_max_mhz": 1965.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# algorithmic work per stage (what the method must do, not what a kernel does)
# ---------------------------------------------------------------------------

def window_keys(N: int, c: int, lookback: int = 1) -> int:
    """sum over queries of the keys in their Sort-LSH window (own chunk and
    ``lookback`` previous ones)."""
    return sum(c * (min((j + 1) * c, N) - max(0, (j - lookback) * c)) for j in range(N // c))


def stage_work(w):
    """Algorithmic work of each stage: (tensor-core flops, HBM bytes).  Bytes
    count what the method must move (inputs read once, outputs written once),
    not what a kernel happens to move; the RACE stages' gathers through L2
    (L d values per row and pass) are not HBM traffic and are not counted."""
    BH, N, d, L, NB = w.B * w.H, w.N, w.d, w.race_tables, 1 << w.race_bits
    e = 2 if w.dtype == "bf16" else 4
    rb = 1 if w.race_bits <= 8 else 2
    P = w.sort_bits + L * w.race_bits
    wk = window_keys(N, w.chunk, w.lookback) * BH   # query-key pairs of the sparse branch
    rows = BH * N
    tables = BH * L * NB
    return {
        "hash": (4.0 * rows * d * P, 2.0 * rows * d * e + 2 * rows * (2 + L * rb)),
        "sort": (0.0, 2.0 * rows * (2 + 4)),
        "race_build": (0.0, rows * (d * e + L * rb) + tables * (4.0 * d + 4)),
        "sparse_fwd": (4.0 * wk * d, rows * (4.0 * d * e + 4 + 8)),
        "race_fuse": (0.0, rows * (4.0 * d * e + L * rb + 8)),
        "fuse_bwd": (0.0, rows * (6.0 * d * e + 24)),
        "race_bwd": (0.0, rows * (d * e + L * rb) + tables * (1.0 * d * e)),
        "sparse_bwd": (10.0 * wk * d, rows * (7.0 * d * e + 24 + 8)),
        "finish": (0.0, rows * (2.0 * d * e + L * rb)),
    }


def stage_roofline(flops, nbytes, sec, peaks):
    """Bound = the resource with the longer ideal time; the tensor peak is the
    sustained one (every stage runs inside a long step)."""
    tf = peaks["bf16_tflops_sustained"] * 1e12
    hb = peaks["hbm_gbs"] * 1e9
    if flops / tf > nbytes / hb:
        ach, peak, unit, bound = flops / sec / 1e12, peaks["bf16_tflops_sustained"], "TFLOP/s", "tensor"
    else:
        ach, peak, unit, bound = nbytes / sec / 1e9, peaks["hbm_gbs"], "GB/s", "hbm"
    return {"bound": bound, "achieved": ach, "peak": peak, "unit": unit, "frac": ach / peak,
            "ideal_us": 1e6 * max(flops / tf, nbytes / hb)}


# DRAM bytes (read + write) of one launch of a stage's main kernel on the
# text-32k workload, from an ncu capture at 12 heads (B=1, H=12) of the same
# source (sha1 of the kernel file); scaled to a launch by the number of
# (batch, head) units, and reported only while that file is unchanged and the
# stage runs the captured kernel (the slab kernels where the path flags say so).
TRAFFIC_WORKLOAD, TRAFFIC_UNITS = "text-32k", 12
RECORDED_TRAFFIC = {
    # stage: (kernel source, its sha1 at capture, bytes per 12-unit launch, path flag needed)
    "hash": ("sparse_rank_hybrid_simhash_b200/csrc/hash_tc.cu", "8587ef1efd310bd3546658819a84be087a7965da", 1.2358e+08, "tc_hash"),
    "race_build": ("sparse_rank_hybrid_simhash_b200/csrc/race.cu", "ae4cba186ff862dc49a580bdd3aa2d9afe804f41", 6.8706e+07, None),
    "sparse_fwd": ("sparse_rank_hybrid_simhash_b200/csrc/attn_tc_pipe.cu", "b33f474224da484dfb1f6128dd2527644c56625a", 1.8644e+08, "tc_attn"),
    "race_fuse": ("sparse_rank_hybrid_simhash_b200/csrc/race_slab.cu", "5135a962ed6cf3d305d45cb27ffcdf41815cc38e", 1.4487e+08, "slab_fwd"),
    "fuse_bwd": ("sparse_rank_hybrid_simhash_b200/csrc/fuse_bwd.cu", "d225c68863731ac35a2126d849af1623d8c512c7", 2.8098e+08, None),
    "race_bwd": ("sparse_rank_hybrid_simhash_b200/csrc/race.cu", "ae4cba186ff862dc49a580bdd3aa2d9afe804f41", 6.6587e+07, None),
    "sparse_bwd": ("sparse_rank_hybrid_simhash_b200/csrc/attn_tc_bwd3.cu", "ffbd2e8b9a9bb8a1a16dfa244ec836a1dc90ccdc", 3.3276e+08, "tc_attn"),
    "finish": ("sparse_rank_hybrid_simhash_b200/csrc/race_slab.cu", "5135a962ed6cf3d305d45cb27ffcdf41815cc38e", 7.874e+07, "slab_bwd"),
}


def recorded_traffic(w, stage, path):
    """DRAM bytes of one full launch of the stage's kernel, or None when the
    capture does not describe what this run launches."""
    rec = RECORDED_TRAFFIC.get(stage)
    ref = WORKLOADS[TRAFFIC_WORKLOAD]
    if rec is None or w.replace(B=ref.B, H=ref.H, seed=ref.seed) != ref:
        return None
    src, sha, nbytes, flag = rec
    if flag is not None and not path.get(flag, False):
        return None
    try:
        with open(os.path.join(ROOT, src), "rb") as f:
            if hashlib.sha1(f.read()).hexdigest() != sha:
                return None
    except OSError:
        return None
    return nbytes * (w.B * w.H) / TRAFFIC_UNITS


def operator_roofline(w, peaks):
    """The whole operator's roofline: max(flops / tensor peak, bytes / HBM peak)."""
    BH, N, d = w.B * w.H, w.N, w.d
    e = 2 if w.dtype == "bf16" else 4
    P = w.sort_bits + w.race_tables * w.race_bits
    wk = window_keys(N, w.chunk, w.lookback) * BH
    rows = BH * N
    f_fwd = 2.0 * 2 * rows * d * P + 4.0 * wk * d
    f_bwd = 10.0 * wk * d
    b_fwd = 4.0 * rows * d * e
    b_all = b_fwd + 2 * (rows * d * e + 8 * rows) + 7.0 * rows * d * e
    tf, hb = peaks["bf16_tflops"] * 1e12, peaks["hbm_gbs"] * 1e9
    return {"fwd_us": 1e6 * max(f_fwd / tf, b_fwd / hb),
            "fwdbwd_us": 1e6 * max((f_fwd + f_bwd) / tf, b_all / hb),
            "flops_fwd": f_fwd, "flops_fwdbwd": f_fwd + f_bwd, "bytes_fwd": b_fwd,
            "bytes_fwdbwd": b_all}


def interaction_count(w):
    """Query-key and query-bucket interactions one step performs ("Two
    Efficient Attentions, One Denominator Problem", section "Linear
    interactions are not yet production economics": the count grows linearly
    in N; the formula itself is lost, the 32K example survives): every query
    scores the keys of its Sort-LSH window (own and previous chunk; with R hash
    rounds at most R windows) and reads one bucket in each of the L RACE
    tables."""
    BH, N = w.B * w.H, w.N
    sparse = window_keys(N, w.chunk, w.lookback) * max(1, w.hash_rounds) / N
    race = w.race_tables
    return {"per_query": sparse + race, "sparse_per_query": sparse, "race_per_query": race,
            "per_step": (sparse + race) * BH * N, "dense_per_query": N,
            "fraction_of_dense": (sparse + race) / N,
            "note": "sparse = window keys (upper bound with several hash rounds), race = L"}


# Stages whose table lines move through on-chip memory, not HBM: every row
# reads (or adds) one line of d values per table.  The gathers of the forward
# read-out and of the value gradient run from shared-memory slabs (where they
# fit); the table builds sum value rows gathered from L2.
RACE_ONCHIP = {"race_build": "l2", "race_fuse": "smem", "race_bwd": "l2", "finish": "smem"}
# measured row-gather rate of an L2-resident table (independent 16-byte loads
# of random 128-byte rows, 592-1184 CTAs on a B200)
L2_GATHER_GBS = 20000.0


def race_onchip_bound(w, stage_ms, sm_mhz, slab_ok):
    """Each RACE stage against its on-chip bound: bytes of table lines per
    pass (rows x L x d x element size of the bf16 tables) over the stage time,
    against shared-memory bandwidth (148 SMs x 128 B per clock x the sampled
    SM clock) for the slab gathers, or the measured L2 row-gather rate."""
    BH, N, d, L = w.B * w.H, w.N, w.d, w.race_tables
    nbytes = BH * N * L * d * 2.0
    smem_gbs = 148 * 128 * (sm_mhz or 1965.0) * 1e6 / 1e9
    out = {}
    for st, kind in RACE_ONCHIP.items():
        if st not in stage_ms or stage_ms[st] <= 0:
            continue
        if kind == "smem" and not slab_ok:
            kind = "l2"
        peak = smem_gbs if kind == "smem" else L2_GATHER_GBS
        ach = nbytes / (stage_ms[st] / 1e3) / 1e9
        out[st] = {"onchip_bytes": nbytes, "achieved_GBs": round(ach, 1),
                   "peak_GBs": round(peak, 1), "frac": round(ach / peak, 4),
                   "peak_kind": ("shared memory: 148 SMs x 128 B/clk x SM clock" if kind == "smem"
                                 else "L2 row gather, measured")}
    return out


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """SM clock and clock-event reasons during the timed region: NVML polled
    every 2 ms from a thread (reading only; nothing is set), else nvidia-smi
    at its 50 ms floor."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int):
        self.proc = None
        self.index = index
        self.samples = []
        self.nvml = None
        self.thread = None
        self.stop = None
        self.out = ""

    def _poll(self):
        nv, h = self.nvml
        while not self.stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((sm, mx, rs))
            except Exception:   # a failed read leaves the sample out
                pass
            time.sleep(0.002)

    def __enter__(self):
        try:
            import pynvml as nv
            import threading
            nv.nvmlInit()
            try:
                idx = torch.cuda._get_nvml_device_index(self.index)
            except Exception:
                idx = self.index
            self.nvml = (nv, nv.nvmlDeviceGetHandleByIndex(idx))
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out = ""
        return False

    def summary(self):
        if self.samples:
            sm = [float(x[0]) for x in self.samples]
            loaded = [v for v in sm if v > 0.5 * max(sm)]
            reasons = sorted({name for x in self.samples for bit, name in self.REASONS.items()
                              if x[2] & bit})
            return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(x[1] for x in self.samples),
                    "reasons": reasons, "samples": len(self.samples), "source": "nvml 2 ms"}
        rows = [r.split(",") for r in self.out.strip().splitlines() if r.count(",") >= 7]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[0]) for r in rows if r[0].strip().replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4)
                          if r[4 + i].strip().lower() == "active"})
        loaded = [v for v in sm if v > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "source": "nvidia-smi 50 ms"}


# ---------------------------------------------------------------------------
# ablation and single-branch modes (same kernels, other gate / lambda settings)
# ---------------------------------------------------------------------------

# mode: (gate_fixed, gate_s, gate_r, lambda or None to keep the workload's)
MODES = {
    "elsaa": None,                          # the workload as drawn: learned gates, lambda = 1
    "sort_lsh_race": (False, None, None, 0.0),   # sparse multiplier fixed to one (lambda = 0)
    "race_only": (True, 0.0, 1.0, None),    # y = O_race
    "sparse_only": (True, 1.0, 0.0, 0.0),   # y = O_sp (Sort-LSH attention alone)
}

STANDS_IN_FOR = {
    "text-32k": "synthetic (seeded; stands in for the ArXiv 32K text task)",
    "vision-16k": "synthetic (seeded; stands in for the 16K image tasks)",
    "needle-256k": "synthetic (seeded; stands in for needle-in-a-haystack)",
}


def bench_config(w, mode, world, l2):
    """The config object of a bench line (both arms)."""
    return {"workload": w.name, "mode": mode, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
            "sort_bits": w.sort_bits, "sort_order": w.sort_order, "lookback": w.lookback,
            "causal": w.causal, "hash_rounds": w.hash_rounds,
            "chunk": w.chunk,
            "race_tables": w.race_tables,
            "race_bits": w.race_bits,
            "gates": "learned" if not w.gate_fixed else f"fixed {w.gate_s}/{w.gate_r}",
            "lambda": w.lam, "global_batch": world * w.B, "seq_len": w.N,
            "parallelism": f"dp{world}", "l2": l2}


def apply_mode(w, mode):
    """The workload with the gate / lambda settings of an ablation mode."""
    m = MODES[mode]
    if m is None:
        return w
    fixed, gs, gr, lam = m
    kw = {"gate_fixed": fixed}
    if gs is not None:
        kw.update(gate_s=gs, gate_r=gr)
    if lam is not None:
        kw["lam"] = lam
    return w.replace(**kw)


def time_dense_sdpa(w, d, steps=3, warmup=2):
    """Dense softmax attention (torch SDPA, its own kernels) forward + backward on
    the same Q, K, V: context for what the sparse branch replaces, not a path of
    this library."""
    import torch.nn.functional as F
    q = d["q"].detach().clone().requires_grad_(True)
    k = d["k"].detach().clone().requires_grad_(True)
    v = d["v"].detach().clone().requires_grad_(True)

    def one():
        o = F.scaled_dot_product_attention(q, k, v)
        o.backward(d["dy"])

    for _ in range(warmup):
        one()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s0.record()
    for _ in range(steps):
        one()
    s1.record()
    torch.cuda.synchronize()
    ms = s0.elapsed_time(s1) / steps
    return {"ms_per_step": ms, "tokens_per_s": w.tokens / (ms / 1e3), "steps": steps,
            "impl": "torch scaled_dot_product_attention (dense, fwd+bwd)"}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args, rank, world, local_rank):
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = apply_mode(WORKLOADS[args.workload], args.mode).replace(
        sort_order=args.sort_order, lookback=args.lookback, causal=args.causal,
        hash_rounds=args.hash_rounds)
    p = B.Params.from_workload(w)
    inp = make_inputs(w, seed=DP.rank_seed(w.seed, rank), with_dy=True)
    d = {k: t.to(dev) for k, t in inp.items()}
    saved = B.alloc_saved(p, dev)
    ws = B.alloc_workspace(p, dev)
    y = torch.empty_like(d["q"])
    grads = [torch.empty_like(d["q"]), torch.empty_like(d["k"]), torch.empty_like(d["v"]),
             torch.empty(2, w.d, dtype=torch.float32, device=dev),
             torch.empty(2, dtype=torch.float32, device=dev),
             torch.empty(1, dtype=torch.float32, device=dev)]
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    nf, nb = len(B.FWD_STAGES), len(B.BWD_STAGES)

    def step(ev_f=None, ev_b=None):
        B.forward(p, d["q"], d["k"], d["v"], d["r_sort"], d["r_race"], d["gate_w"], d["gate_b"],
                  d["lam"], y=y, saved=saved, ws=ws, events=ev_f)
        B.backward(p, d["q"], d["k"], d["v"], d["r_sort"], d["r_race"], d["gate_w"],
                   d["gate_b"], d["lam"], saved, d["dy"], *grads, ws=ws, events=ev_b)
        if world > 1:
            DP.allreduce_param_grads(grads[3], grads[4], grads[5])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    B.check(ws)

    mk = lambda: torch.cuda.Event(enable_timing=True)
    evs = [([mk() for _ in range(nf + 1)], [mk() for _ in range(nb + 1)], mk())
           for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)            # L2 flush between timed steps, outside the events
            ef, eb, end = evs[i]
            step(ef, eb)
            end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    B.check(ws)
    step_ms = [ef[0].elapsed_time(end) for ef, eb, end in evs]
    fwd_ms = [ef[0].elapsed_time(ef[-1]) for ef, eb, end in evs]
    stage_ms = {}
    for j, name in enumerate(B.FWD_STAGES):
        stage_ms[name] = statistics.mean(ef[j].elapsed_time(ef[j + 1]) for ef, eb, end in evs)
    for j, name in enumerate(B.BWD_STAGES):
        stage_ms[name] = statistics.mean(eb[j].elapsed_time(eb[j + 1]) for ef, eb, end in evs)
    total_ms = sum(step_ms)
    fwd_total = sum(fwd_ms)
    if world > 1:
        total_ms, fwd_total = DP.max_over_ranks([total_ms, fwd_total], dev)

    views = B.saved_views(p, saved)
    dev_unit = {"y": y[0, 0].cpu()}
    dev_unit.update({k: views[k][0, 0].cpu() for k in ("code_q", "code_k", "rcode_q", "rcode_k")})
    del saved, ws, grads, flush
    torch.cuda.empty_cache()
    # end to end through the public API with host buffers
    e2e = run_e2e(args, w, p, inp, dev, world)
    context = time_dense_sdpa(w, d) if args.dense_context and world == 1 else None
    return w, p, total_ms, fwd_total, stage_ms, clk.summary(), e2e, context, dev_unit


def run_e2e(args, w, p, inp, dev, world):
    """The same step end to end through the public API with host buffers: the
    batch's inputs sit in pinned host memory and its outputs go back there
    every step, streamed through the device in groups of heads
    (pipeline.HostStepPipeline: copy-in, compute and copy-out overlap)."""
    from sparse_rank_hybrid_simhash_b200.pipeline import HostStepPipeline
    BH = w.B * w.H
    # more groups shorten the unoverlapped first copy-in and last copy-out
    groups = next(g for g in (8, 6, 4, 3, 2, 1) if BH % g == 0)
    host = {k: inp[k].pin_memory() for k in ("q", "k", "v", "dy")}
    outs = {k: torch.empty_like(host["q"], pin_memory=True) for k in ("y", "dq", "dk", "dv")}
    pipe = HostStepPipeline(p, groups, dev, inp["r_sort"], inp["r_race"], inp["gate_w"],
                            inp["gate_b"], inp["lam"])
    stream = torch.cuda.current_stream()
    pg_dev = torch.empty(2 * w.d + 3, dtype=torch.float32, device=dev)

    def step():
        if world > 1:   # the shared-parameter gradients, summed over ranks, every step
            pipe.enqueue(host, outs, stream)
            stream.synchronize()
            gw, gb, gl = pipe.gradients()
            pg_dev.copy_(torch.cat([gw.view(-1), gb, gl]))
            torch.distributed.all_reduce(pg_dev)
        else:           # back to back: a step's copy-in overlaps the last one's tail
            pipe.enqueue_chained(host, outs)

    step()
    pipe.join(stream)
    torch.cuda.synchronize()
    n = max(3, min(args.steps, 10))
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    start.record(stream)
    pipe.start_after(stream)
    for _ in range(n):
        step()
    pipe.join(stream)
    end.record(stream)
    torch.cuda.synchronize()
    pipe.gradients()
    ms = start.elapsed_time(end)
    if world > 1:
        ms = DP.max_over_ranks([ms], dev)[0]
    h2d = pipe.h2d_bytes(host)
    d2h = sum(t.numel() * t.element_size() for t in outs.values()) + pipe.pg_host.numel() * 4
    return {"value": world * n * w.tokens / (ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n,
            "pipeline": f"{groups} head groups; copy-in, compute and copy-out streams overlap"
                        + ("" if world > 1 else ", consecutive steps too")}


# ---------------------------------------------------------------------------
# a sequence split over ranks (shard.py)
# ---------------------------------------------------------------------------

def run_seq_shards(args, rank, world, local_rank):
    """Forward (and backward where the workload has one) of one workload with
    every unit's sequence split into args.seq_shards token shards: one shard
    per rank under torchrun (NCCL collectives), or every shard in this process
    on one GPU (the collectives become device copies: an emulation of the
    split, all shards' work serialised).  Total work is fixed (strong scaling)."""
    from sparse_rank_hybrid_simhash_b200.shard import DistComm, LocalComm, ShardedElsaa
    P = args.seq_shards
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    p = B.Params.from_workload(w)
    if world > 1:
        if world != P:
            raise SystemExit("--seq-shards must equal the number of ranks")
        comm, mine = DistComm(), [rank]
    else:
        comm, mine = LocalComm(P), list(range(P))
    inp = make_inputs(w, with_dy=w.backward)
    M = w.N // P
    sh = {n: [inp[n][:, :, r * M:(r + 1) * M].contiguous().to(dev) for r in mine]
          for n in (("q", "k", "v", "dy") if w.backward else ("q", "k", "v"))}
    args_ = tuple(inp[n].to(dev) for n in ("r_sort", "r_race", "gate_w", "gate_b", "lam"))
    op = ShardedElsaa(p, comm)

    def step():
        op.forward(sh["q"], sh["k"], sh["v"], *args_)
        if w.backward:
            op.backward(sh["dy"], *args_)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(args.steps):
        step()
    end.record()
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    if world > 1:
        ms = DP.max_over_ranks([ms], dev)[0]
    if rank == 0:
        line = {
            "metric": f"ELSAA tokens/s, {w.name} sequence split over {P} shards "
                      + ("(fwd+bwd)" if w.backward else "(fwd)"),
            "value": args.steps * w.tokens / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": w.dtype, "data": STANDS_IN_FOR.get(w.name, "synthetic (seeded)"),
            "config": dict(bench_config(w, "elsaa", world, "inputs > L2"), seq_shards=P,
                           parallelism=f"sequence split x{P}"),
            "emulated": world == 1 and P > 1,
            "note": ("all shards in one process on one GPU: collectives are device copies and "
                     "the shards' work is serialised" if world == 1 and P > 1 else
                     "one shard per rank, NCCL all-gather / all-to-all / all-reduce"),
        }
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# the other workloads, device-timed (context for the headline)
# ---------------------------------------------------------------------------

def time_workload(name, dev, steps=5, warmup=3):
    """Forward (and forward + backward where the workload has one) of another
    workload at full size, device-timed with CUDA events and an L2 flush
    between steps; tokens/s and the operator-roofline fractions."""
    w = WORKLOADS[name]
    p = B.Params.from_workload(w)
    d = {k: t.to(dev) for k, t in make_inputs(w, with_dy=w.backward).items()}
    saved = B.alloc_saved(p, dev)
    ws = B.alloc_workspace(p, dev)
    y = torch.empty_like(d["q"])
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def fwd():
        B.forward(p, d["q"], d["k"], d["v"], d["r_sort"], d["r_race"], d["gate_w"],
                  d["gate_b"], d["lam"], y=y, saved=saved, ws=ws)

    def bwd():
        B.backward(p, d["q"], d["k"], d["v"], d["r_sort"], d["r_race"], d["gate_w"],
                   d["gate_b"], d["lam"], saved, d["dy"], ws=ws)

    for _ in range(warmup):
        fwd()
        if w.backward:
            bwd()
    torch.cuda.synchronize()
    B.check(ws)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for e in ev:
        flush.fill_(1)
        e[0].record()
        fwd()
        e[1].record()
        if w.backward:
            bwd()
        e[2].record()
    torch.cuda.synchronize()
    B.check(ws)
    peaks = load_peaks()
    roof = operator_roofline(w, peaks)
    f_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    out = {"shape": f"B{w.B} H{w.H} N{w.N} d{w.d} {w.dtype}", "fwd_ms": round(f_ms, 4),
           "fwd_tokens_per_s": w.tokens / (f_ms / 1e3),
           "fwd_roofline_us": round(roof["fwd_us"], 2),
           "fwd_roofline_frac": roof["fwd_us"] / (1e3 * f_ms),
           "path": B.path_flags(p), "steps": steps}
    if w.backward:
        fb_ms = statistics.mean(e[0].elapsed_time(e[2]) for e in ev)
        out.update({"fwdbwd_ms": round(fb_ms, 4), "fwdbwd_tokens_per_s": w.tokens / (fb_ms / 1e3),
                    "fwdbwd_roofline_us": round(roof["fwdbwd_us"], 2),
                    "fwdbwd_roofline_frac": roof["fwdbwd_us"] / (1e3 * fb_ms)})
    del d, saved, ws, y, flush
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------------
# the oracle as CPU baseline and as the reference arm
# ---------------------------------------------------------------------------

def oracle_unit_seconds(w, inp, units):
    import oracle as O
    t0 = time.perf_counter()
    for (b, h) in units:
        args = (inp["q"][b, h], inp["k"][b, h], inp["v"][b, h], inp["r_sort"], inp["r_race"],
                w.chunk)
        fixed = (w.gate_s, w.gate_r) if w.gate_fixed else None
        O.grads_head(*args, inp["dy"][b, h], None, inp["gate_w"], inp["gate_b"],
                     float(inp["lam"][0]), fixed, sort_order=w.sort_order,
                     lookback=w.lookback, causal=w.causal)
    return time.perf_counter() - t0


def cpu_baseline(w, min_seconds=10.0, device_unit=None):
    """The oracle on the host cores over (batch, head) units of the workload,
    one after another until at least min_seconds of CPU work (or every unit).
    With ``device_unit`` (unit (0, 0) of the timed device run: y and the
    codes), the oracle's forward of that unit also gives the parity figures of
    the bench line (outside the timed oracle calls)."""
    cores = len(os.sched_getaffinity(0))
    torch.set_num_threads(cores)
    inp = make_inputs(w, with_dy=True)
    all_units = [(i // w.H % w.B, i % w.H) for i in range(w.B * w.H)]
    secs, units = 0.0, 0
    while units < len(all_units) and secs < min_seconds:
        secs += oracle_unit_seconds(w, inp, all_units[units:units + 1])
        units += 1
    # one (batch, head) unit is N / H token-equivalents of the B x N-token step
    value = units * w.N / w.H / secs
    out = {"value": value, "unit": "tokens/s", "cores": torch.get_num_threads(),
           "kind": "oracle",
           "sample": f"{units} of {w.B * w.H} (batch, head) units of {w.name}, forward+backward "
                     f"in fp64 ({secs:.1f} s), scaled to the whole step"}
    if device_unit is not None:
        out["parity_unit"] = parity_sample(w, inp, device_unit)
    return out


def parity_sample(w, inp, dev_unit):
    """Unit (0, 0) of the timed run against the oracle: code mismatches, codes
    whose projection lies within rounding of zero, and rel-L2 / max-abs of y."""
    import oracle as O
    fixed = (w.gate_s, w.gate_r) if w.gate_fixed else None
    ref = O.forward_head(inp["q"][0, 0], inp["k"][0, 0], inp["v"][0, 0], inp["r_sort"],
                         inp["r_race"], w.chunk, None, inp["gate_w"], inp["gate_b"],
                         float(inp["lam"][0]), fixed, sort_order=w.sort_order,
                         lookback=w.lookback, causal=w.causal)
    mism, near, total = 0, 0, 0
    for key in ("code_q", "code_k", "rcode_q", "rcode_k"):
        got = dev_unit[key].to(torch.int64) & 0xFFFF
        mism += int((got != ref[key]).sum())
        near += int(ref["near_" + key].sum())
        total += ref[key].numel()
    y, ry = dev_unit["y"].double(), ref["y"]
    return {"unit": "(0, 0)", "codes": total, "code_mismatches": mism,
            "near_zero_projections": near, "y_rel_l2": float((y - ry).norm() / ry.norm()),
            "y_max_abs": float((y - ry).abs().max())}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = apply_mode(WORKLOADS[args.workload], args.mode).replace(
        sort_order=args.sort_order, lookback=args.lookback, causal=args.causal,
        hash_rounds=args.hash_rounds)
    cores = len(os.sched_getaffinity(0))
    torch.set_num_threads(cores)
    inp = make_inputs(w, with_dy=True)
    per_step = 2
    units = [(i // w.H % w.B, i % w.H) for i in range(w.B * w.H)]
    for i in range(args.warmup):
        oracle_unit_seconds(w, inp, units[:1])
    secs = []
    for i in range(args.steps):
        sel = [units[(i * per_step + j) % len(units)] for j in range(per_step)]
        secs.append(oracle_unit_seconds(w, inp, sel))
    total = sum(secs)
    value = args.steps * per_step * w.N / w.H / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps * (w.B * w.H / per_step),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": STANDS_IN_FOR.get(w.name, "synthetic (seeded)"),
        "config": bench_config(w, args.mode, args.gpus, "n/a (CPU)"),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": torch.get_num_threads(),
                         "kind": "oracle",
                         "sample": f"{per_step} of {w.B * w.H} (batch, head) units per step, "
                                   "forward+backward in fp64, scaled to the whole step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the device timing of iid-4k, vision-16k and needle-256k")
    ap.add_argument("--mode", default="elsaa", choices=sorted(MODES),
                    help="ablation / single-branch setting of the gates and lambda")
    ap.add_argument("--sort-order", default="binary", choices=["binary", "gray", "local"],
                    help="Sort-LSH chunk order: code value, Gray sequence, or token order")
    ap.add_argument("--lookback", type=int, default=1,
                    help="previous sorted chunks a query chunk attends (1: own and previous)")
    ap.add_argument("--hash-rounds", type=int, default=1,
                    help="Sort-LSH hash rounds; a query attends the union of its windows")
    ap.add_argument("--causal", action="store_true",
                    help="keys j <= i only (CUDA-core attention, RACE token scans)")
    ap.add_argument("--dense-context", action="store_true",
                    help="also time dense torch SDPA fwd+bwd on the same inputs (context)")
    ap.add_argument("--seq-shards", type=int, default=0,
                    help="split every unit's sequence into this many token shards (one per "
                         "rank under torchrun; all in this process on one GPU)")
    ap.add_argument("--batch", type=int, default=None,
                    help="override B (small cases for ncu captures; not a bench line)")
    ap.add_argument("--heads", type=int, default=None,
                    help="override H (small cases for ncu captures; not a bench line)")
    args = ap.parse_args()
    if args.batch or args.heads:
        w0 = WORKLOADS[args.workload]
        WORKLOADS[args.workload] = w0.replace(B=args.batch or w0.B, H=args.heads or w0.H)
    if args.impl == "reference":
        run_reference(args)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    if args.seq_shards:
        run_seq_shards(args, rank, world, local_rank)
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        return
    w, p, total_ms, fwd_ms, stage_ms, clocks, e2e, context, dev_unit = run_ours(
        args, rank, world, local_rank)
    peaks = load_peaks()
    if rank == 0:
        K = args.steps
        value = world * K * w.tokens / (total_ms / 1e3)
        fwd_value = world * K * w.tokens / (fwd_ms / 1e3)
        work = stage_work(w)
        per_stage = {st: stage_roofline(*work[st], stage_ms[st] / 1e3, peaks)
                     for st in stage_ms}
        dom = max(stage_ms, key=lambda st: stage_ms[st])
        rl = per_stage[dom]
        path = B.path_flags(p)
        traffic = recorded_traffic(w, dom, path)
        roof = operator_roofline(w, peaks)
        fwd_launch, bwd_launch = B.kernel_launches(p)
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": STANDS_IN_FOR.get(w.name, "synthetic (seeded)"),
            "config": bench_config(w, args.mode, world,
                                   "256 MB flush between timed steps; inputs 0.4 GB > L2"),
            "fwd_tokens_per_s": fwd_value,
            "stages_ms": {k: round(v, 4) for k, v in stage_ms.items()},
            "roofline": {"bound": rl["bound"], "kernel": dom, "achieved": rl["achieved"],
                         "peak": rl["peak"], "unit": rl["unit"], "frac": rl["frac"],
                         "traffic": traffic,
                         "peak_source": peaks["source"] + (" sustained" if rl["bound"] == "tensor"
                                                           else "")},
            "stage_roofline": {st: dict({k: (round(v, 4) if isinstance(v, float) else v)
                                         for k, v in r.items()},
                                        traffic=recorded_traffic(w, st, path))
                               for st, r in per_stage.items()},
            "operator_roofline": {
                "fwd_us": roof["fwd_us"], "fwdbwd_us": roof["fwdbwd_us"],
                "frac_fwd": roof["fwd_us"] / (1e3 * fwd_ms / K),
                "frac_fwdbwd": roof["fwdbwd_us"] / (1e3 * total_ms / K)},
            "gpu_launches": K * (fwd_launch + bwd_launch),
            "clocks": clocks,
            "e2e": e2e,
        }
        line["interactions"] = interaction_count(w)
        line["race_onchip"] = race_onchip_bound(w, stage_ms, clocks.get("sm_mhz"),
                                                path["slab_fwd"])
        line["path"] = path
        if context is not None:
            line["context"] = {"dense_sdpa": context}
        if world == 1 and not args.no_other_workloads and args.workload == WORKLOAD:
            line["other_workloads"] = {name: time_workload(name, torch.device("cuda", local_rank))
                                       for name in ("iid-4k", "vision-16k", "needle-256k")}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w, device_unit=dev_unit)
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
