"""GPU parity: the C-ABI path against the fp64 oracle on the same seeded inputs.

Small cases span several chunks, several 128-row tiles and a ragged tail of
the radix-sort tiles; every unit and every saved intermediate is compared.
"""

import pytest
import torch

from sparse_rank_hybrid_simhash_b200 import binding as B
from sparse_rank_hybrid_simhash_b200.workloads import WORKLOADS, make_inputs, small

from parity import check_param_grads, check_unit, run_gpu

pytestmark = pytest.mark.gpu


def _all_units(w):
    return [(b, h) for b in range(w.B) for h in range(w.H)]


def _run(w, backward, report=None):
    inp = make_inputs(w, with_dy=backward)
    gpu = run_gpu(w, inp, backward)
    report = {} if report is None else report
    refs = [check_unit(w, inp, gpu, b, h, backward, report) for (b, h) in _all_units(w)]
    if backward:
        check_param_grads(w, gpu, refs)
    return report


def test_tiny_fp32_forward_full_size(cuda_device):
    _run(WORKLOADS["tiny-fp32"], backward=False)


def test_tiny_fp32_backward(cuda_device):
    _run(WORKLOADS["tiny-fp32"].replace(gate_fixed=False), backward=True)


@pytest.mark.parametrize("name", ["iid-4k", "vision-16k", "text-32k"])
def test_small_forward_backward(cuda_device, name):
    w = small(WORKLOADS[name], B=1, H=2, N=1024)
    _run(w, backward=True)


def test_needle_small_forward(cuda_device):
    w = small(WORKLOADS["needle-256k"], B=1, H=2, N=2048)
    _run(w, backward=False)


@pytest.mark.parametrize("d,N,L,kr,sort_bits,chunk", [
    (64, 960, 12, 5, 6, 64),      # N not a multiple of 128: tiles straddle units
    (128, 640, 5, 9, 11, 128),    # 16-bit codes, 10 bytes of codes per row
    (64, 1024, 3, 13, 1, 64),     # 16-bit codes, 6 bytes per row, 8192 buckets
    (128, 1088, 20, 7, 8, 64),    # two passes (148 columns), ragged N
    (64, 512, 3, 0, 5, 64),       # no RACE bits (one bucket): sort codes only
    (64, 576, 6, 4, 0, 64),       # no sort bits: every code from the RACE columns
])
def test_bit_stream_hash_shapes(cuda_device, d, N, L, kr, sort_bits, chunk):
    # shapes the word-aligned hash layout does not take (row codes not whole
    # 32-bit words, or N not a multiple of 128): the bit-stream tcgen05 hash,
    # with codes cut across word boundaries; every code compared
    w = small(WORKLOADS["iid-4k"], B=2, H=2, N=N).replace(
        d=d, race_tables=L, race_bits=kr, sort_bits=sort_bits, chunk=chunk, backward=False)
    assert B.path_flags(B.Params.from_workload(w))["tc_hash"]
    _run(w, backward=False)


def test_bit_stream_hash_many_tiles_per_cta(cuda_device):
    # 2056 tiles of 128 rows: every CTA of the bit-stream hash takes several,
    # so both bit arrays and both handovers between its readers and writers
    # are used; N is not a multiple of 128, so tiles straddle units
    w = small(WORKLOADS["iid-4k"], B=2, H=4, N=16448).replace(
        race_tables=12, race_bits=5, sort_bits=6, chunk=64, backward=False)
    inp = make_inputs(w, with_dy=False)
    gpu = run_gpu(w, inp, backward=False)
    for b, h in [(0, 0), (1, 3)]:
        check_unit(w, inp, gpu, b, h, False, {})


@pytest.mark.parametrize("lam,gates", [(0.0, (1.0, 0.0)), (2.0, (0.0, 1.0)), (0.0, (0.3, 0.9))])
def test_ablation_and_single_branch_modes(cuda_device, lam, gates):
    w = small(WORKLOADS["iid-4k"], B=1, H=2, N=512).replace(
        gate_fixed=True, gate_s=gates[0], gate_r=gates[1], lam=lam)
    _run(w, backward=True)


@pytest.mark.parametrize("N,chunk", [(64, 64), (192, 64), (320, 32), (2048 + 64, 64)])
def test_single_chunk_and_ragged_lengths(cuda_device, N, chunk):
    # one chunk (dense attention), lengths that are not multiples of 128 or of
    # the 2048-key sort tile
    w = WORKLOADS["iid-4k"].replace(B=1, H=2, N=N, chunk=chunk)
    _run(w, backward=True)


@pytest.mark.parametrize("chunk", [16, 32])
def test_small_chunks(cuda_device, chunk):
    # windows narrower than the 128-row tiles: the attention kernels mask by chunk
    w = WORKLOADS["iid-4k"].replace(B=1, H=2, N=1024, chunk=chunk)
    _run(w, backward=True)


@pytest.mark.parametrize("order,sort_bits", [("gray", 7), ("gray", 12), ("local", 4)])
def test_sort_orders(cuda_device, order, sort_bits):
    # Gray-sequence bucket order (one and two radix passes) and local windows
    # in token order, through the same attention and RACE kernels
    w = WORKLOADS["iid-4k"].replace(B=1, H=2, N=1024, chunk=64, sort_bits=sort_bits,
                                    sort_order=order)
    _run(w, backward=True)


@pytest.mark.parametrize("rounds,dtype,order,causal", [(2, "bf16", "binary", False),
                                                       (3, "bf16", "gray", False),
                                                       (3, "f32", "binary", True)])
def test_hash_rounds(cuda_device, rounds, dtype, order, causal):
    # several Sort-LSH hash rounds: every round's codes and orders, and the
    # attention over the union of the rounds' windows (each key once)
    w = WORKLOADS["iid-4k"].replace(B=1, H=2, N=512, chunk=32, dtype=dtype, sort_order=order,
                                    causal=causal, hash_rounds=rounds)
    _run(w, backward=True)


@pytest.mark.parametrize("rounds,d,N,chunk,lookback,causal", [
    (2, 64, 2048, 128, 1, False), (4, 64, 1024, 64, 2, False), (2, 128, 1024, 256, 0, False),
    (3, 64, 1024, 32, 1, True), (8, 64, 512, 64, 1, False)])
def test_hash_rounds_tensor_cores(cuda_device, rounds, d, N, chunk, lookback, causal):
    # several rounds in bf16: one streamed-window pass per round, keys of an
    # earlier round's window masked, partial softmaxes combined; backward one
    # key-major pass per round with the final lse
    w = WORKLOADS["iid-4k"].replace(B=1, H=2, N=N, d=d, chunk=chunk, lookback=lookback,
                                    causal=causal, hash_rounds=rounds)
    f = B.path_flags(B.Params.from_workload(w))
    assert f["tc_win"] and f["tc_attn"]
    _run(w, backward=True)


@pytest.mark.parametrize("lookback,dtype,chunk,N", [(0, "bf16", 32, 512), (2, "bf16", 32, 512),
                                                    (3, "f32", 32, 512), (2, "bf16", 128, 2048),
                                                    (4, "bf16", 64, 1024)])
def test_lookback(cuda_device, lookback, dtype, chunk, N):
    # windows of lookback previous chunks plus the own one: bf16 on the
    # streamed-window forward and the key-major tcgen05 backward, fp32 on the
    # CUDA-core attention
    w = WORKLOADS["iid-4k"].replace(B=1, H=2, N=N, chunk=chunk, lookback=lookback, dtype=dtype)
    assert B.path_flags(B.Params.from_workload(w))["tc_attn"] == (dtype == "bf16")
    _run(w, backward=True)


@pytest.mark.parametrize("d,N,chunk,lookback", [(64, 2048, 256, 1), (128, 1024, 128, 1),
                                                (128, 1024, 64, 3), (64, 1536, 384, 1),
                                                (64, 1152, 96, 2), (128, 2048, 256, 0)])
def test_streamed_window_forward(cuda_device, d, N, chunk, lookback):
    # the tcgen05 forward that streams each tile's window in 128-key blocks:
    # chunks above 128 (unmasked, several blocks), d = 128, lookback other
    # than 1, and chunks that neither divide nor are multiples of 128 (masked)
    w = WORKLOADS["iid-4k"].replace(B=1, H=2, N=N, d=d, chunk=chunk, lookback=lookback)
    assert B.path_flags(B.Params.from_workload(w))["tc_win"]
    _run(w, backward=True)


@pytest.mark.parametrize("dtype,order,gates,d,N,chunk,lookback", [
    ("bf16", "binary", False, 64, 512, 32, 1), ("f32", "local", False, 64, 512, 32, 1),
    ("bf16", "binary", True, 64, 512, 32, 1), ("bf16", "gray", False, 64, 2048, 128, 1),
    ("bf16", "binary", False, 128, 1024, 64, 2), ("bf16", "local", False, 64, 1024, 256, 0)])
def test_causal(cuda_device, dtype, order, gates, d, N, chunk, lookback):
    # keys j <= i in both branches (per-table RACE token scans; bf16 on the
    # streamed-window forward and the key-major tcgen05 backward, fp32 on the
    # CUDA-core attention); binary order leaves some early queries with empty
    # windows
    w = WORKLOADS["iid-4k"].replace(B=1, H=2, N=N, d=d, chunk=chunk, lookback=lookback,
                                    dtype=dtype, sort_order=order, causal=True,
                                    gate_fixed=gates, gate_s=0.6, gate_r=0.8)
    assert B.path_flags(B.Params.from_workload(w))["tc_win"] == (dtype == "bf16")
    _run(w, backward=True)


@pytest.mark.parametrize("tables,race_bits,N", [(12, 6, 512), (16, 6, 512 + 16), (8, 9, 512),
                                               (4, 6, 256)])
def test_causal_race_walks(cuda_device, tables, race_bits, N):
    # the causal RACE read-out and value gradient: the warp walk over 32-token
    # groups (4, 8 and 16 tables; 16-bit codes at 9 bits), and the per-table
    # token scans where the walk does not apply (12 tables; a length that is
    # not a multiple of 32)
    w = WORKLOADS["iid-4k"].replace(B=1, H=2, N=N, chunk=16 if N % 32 else 32,
                                    race_tables=tables, race_bits=race_bits, causal=True)
    _run(w, backward=True)


def test_two_pass_sort_and_wide_race_codes(cuda_device):
    # 12 sort bits take two radix passes; 11 RACE bits give uint16 codes and
    # 2048-bucket tables (the global-atomic build)
    w = WORKLOADS["iid-4k"].replace(B=1, H=1, N=1024, sort_bits=12, race_bits=11,
                                    race_tables=3, chunk=64)
    _run(w, backward=True)


def test_zero_race_bits(cuda_device):
    w = WORKLOADS["iid-4k"].replace(B=1, H=1, N=512, race_bits=0, chunk=64)
    _run(w, backward=True)


@pytest.mark.parametrize("name", ["text-32k", "vision-16k"])
def test_bitwise_reproducible(cuda_device, name):
    """Two runs on the same inputs give identical bits: every reduction in the
    path (table builds, sums, atomics into accumulators) has a fixed order or
    is exact."""
    w = small(WORKLOADS[name], B=1, H=2, N=4096)
    inp = make_inputs(w, with_dy=True)
    a = run_gpu(w, inp, backward=True)
    b = run_gpu(w, inp, backward=True)
    for key in ("y", "dq", "dk", "dv", "dgate_w", "dgate_b", "dlambda"):
        assert torch.equal(a[key], b[key]), key
    for key in ("race_sum", "race_count", "lse_sp", "o_sp", "o_race"):
        assert torch.equal(a["views"][key], b["views"][key]), key
