"""The C ABI without a GPU: the library loads, exports every declared symbol,
and its host-side validation and sizing behave as include/elsaa.h states."""

import ctypes
import os
import re

import pytest

from sparse_rank_hybrid_simhash_b200 import binding as B
from sparse_rank_hybrid_simhash_b200.workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "elsaa.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(elsaa_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = B.lib()
    names = declared_functions()
    assert "elsaa_forward" in names and "elsaa_backward" in names
    for name in names:
        assert hasattr(lib, name), name
    assert set(B.EXPORTS) <= set(names)


def test_params_struct_matches_header_field_order():
    text = open(HEADER).read()
    body = text[text.index("typedef struct {"):text.index("} elsaa_params;")]
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    fields = []
    for decl in body.split(";"):
        decl = decl.replace("typedef struct {", "").strip()
        if not decl:
            continue
        names = decl.split(None, 1)[1]
        fields += [n.strip() for n in names.split(",")]
    assert fields == [f[0] for f in B.Params._fields_]


def test_status_strings():
    lib = B.lib()
    for code, text in B.STATUS.items():
        assert lib.elsaa_status_str(code).decode() == text


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_workloads_validate_and_size(name):
    w = WORKLOADS[name]
    p = B.Params.from_workload(w)
    assert B.validate(p) == 0
    bhn = w.B * w.H * w.N
    esz = 2 if w.dtype == "bf16" else 4
    saved = B.saved_bytes(p)
    # codes, perms, RACE codes (row-major and table-major), tables, lse, O_sp, O_race, Ctot
    expect = (2 * bhn * 2 + 2 * bhn * 4 + 4 * bhn * w.race_tables * (1 if w.race_bits <= 8 else 2)
              + w.B * w.H * w.race_tables * (1 << w.race_bits) * (4 + 4 * w.d)
              + bhn * 4 * 2 + 2 * bhn * w.d * esz)
    assert expect <= saved <= expect + 256 * 16
    assert B.workspace_bytes(p) >= saved


def test_validation_rejects_bad_problems():
    good = B.Params.make(1, 2, 256, 64, "bf16", 4, 64, 8, 6)
    assert B.validate(good) == 0
    cases = [
        dict(N=250),                 # N not a multiple of the chunk
        dict(chunk=0),
        dict(d=0),
        dict(sort_bits=17),
        dict(race_bits=17),
        dict(race_tables=0),
        dict(dtype=7),
        dict(sort_order=3),
        dict(sort_order=-1),
        dict(lookback=-1),
        dict(lookback=65),
        dict(causal=2),
        dict(hash_rounds=-1),
        dict(hash_rounds=9),
        dict(N=0),                   # empty sequence
        dict(B=0),
        dict(H=-1),
        dict(B=1 << 20, H=1 << 10),  # more than 2^40 elements
    ]
    for c in cases:
        p = B.Params.make(1, 2, 256, 64, "bf16", 4, 64, 8, 6)
        for k, v in c.items():
            setattr(p, k, v)
        assert B.validate(p) == 1, c
        assert B.workspace_bytes(p) == 0 and B.saved_bytes(p) == 0
    p = B.Params.make(1, 2, 256, 48, "bf16", 4, 64, 8, 6)   # head dim not a multiple of 32
    assert B.validate(p) == 2
    for order in B.SORT_ORDERS:
        assert B.validate(B.Params.make(1, 2, 256, 64, "bf16", 4, 64, 8, 6, sort_order=order)) == 0
    for lb in (0, 1, 3):
        assert B.validate(B.Params.make(1, 2, 256, 64, "bf16", 4, 64, 8, 6, lookback=lb)) == 0
    # the CUDA-core attention keeps (lookback + 1) chunk scores per query in shared memory
    p = B.Params.make(1, 2, 8192, 64, "bf16", 4, 1024, 8, 6, lookback=6)
    assert B.validate(p) == 2
    assert B.validate(B.Params.make(1, 2, 256, 64, "bf16", 4, 64, 8, 8, causal=True)) == 0
    # several hash rounds: R windows of scores per query in shared memory
    for r in (0, 1, 2, 8):
        assert B.validate(B.Params.make(1, 2, 256, 64, "bf16", 4, 64, 8, 6, hash_rounds=r)) == 0
    assert B.validate(B.Params.make(1, 2, 8192, 64, "bf16", 4, 1024, 8, 6, hash_rounds=4)) == 2
    # one round: 0 and 1 are the same problem with the same saved layout
    p0 = B.Params.make(1, 2, 256, 64, "bf16", 4, 64, 8, 6, hash_rounds=0)
    p1 = B.Params.make(1, 2, 256, 64, "bf16", 4, 64, 8, 6, hash_rounds=1)
    assert B.saved_bytes(p0) == B.saved_bytes(p1)
    p3 = B.Params.make(1, 2, 256, 64, "bf16", 4, 64, 8, 6, hash_rounds=3)
    # codes, orders and inverse orders of two more rounds
    assert B.saved_bytes(p3) >= B.saved_bytes(p1) + 2 * 2 * 512 * (2 + 4) + 3 * 2 * 512 * 4
    # the causal RACE walk keeps a column slab of every table in shared memory
    # (L dividing 32); other table counts take the per-table scan, which keeps
    # one whole table there
    assert B.validate(B.Params.make(1, 2, 256, 128, "bf16", 4, 64, 8, 9, causal=True)) == 0
    assert B.validate(B.Params.make(1, 2, 256, 128, "bf16", 4, 64, 12, 9, causal=True)) == 2
    assert B.validate(B.Params.make(1, 2, 256, 128, "bf16", 4, 64, 12, 8, causal=True)) == 0


def test_null_pointers_are_rejected_before_any_launch():
    p = B.Params.make(1, 1, 256, 64, "bf16", 4, 64, 8, 6)
    lib = B.lib()
    null = ctypes.c_void_p(None)
    code = lib.elsaa_forward(ctypes.byref(p), *([null] * 10), null, 0, null)
    assert code == 1
    code = lib.elsaa_backward(ctypes.byref(p), *([null] * 17), 0, null)
    assert code == 1
    assert lib.elsaa_check(null, null) == 1


def test_workspace_too_small_is_reported():
    p = B.Params.make(1, 1, 256, 64, "bf16", 4, 64, 8, 6, gate_fixed=True)
    lib = B.lib()
    fake = ctypes.c_void_p(1 << 20)   # aligned, never dereferenced: validation fails first
    args = [fake] * 5 + [ctypes.c_void_p(None)] * 2 + [fake, fake, ctypes.c_void_p(None)]
    code = lib.elsaa_forward(ctypes.byref(p), *args, fake, B.workspace_bytes(p) - 256,
                             ctypes.c_void_p(None))
    assert code == 3


def test_misaligned_buffers_are_rejected():
    p = B.Params.make(1, 1, 256, 64, "bf16", 4, 64, 8, 6, gate_fixed=True)
    lib = B.lib()
    good, bad = ctypes.c_void_p(1 << 20), ctypes.c_void_p((1 << 20) + 8)
    args = [bad] + [good] * 4 + [ctypes.c_void_p(None)] * 2 + [good, good, ctypes.c_void_p(None)]
    code = lib.elsaa_forward(ctypes.byref(p), *args, good, B.workspace_bytes(p),
                             ctypes.c_void_p(None))
    assert code == 1


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_tensor_core_path_selection(name):
    w = WORKLOADS[name]
    expect = w.dtype == "bf16"   # every bf16 workload tiles onto the tcgen05 kernels
    assert B.uses_tensor_cores(B.Params.from_workload(w)) == expect
    if expect:
        # and so do its extensions: other lookbacks, the causal mask, several rounds
        # (where the library accepts them: causal needle-256k's 64 x 1024-bucket
        # tables fit neither causal RACE kernel and are rejected)
        for x in (w.replace(lookback=2), w.replace(causal=True), w.replace(hash_rounds=2)):
            p = B.Params.from_workload(x)
            if B.validate(p) == 0:
                assert B.uses_tensor_cores(p) == 1, x
            else:
                assert x.causal and x.race_tables > 32 and B.uses_tensor_cores(p) == 0


def test_kernel_launch_counts():
    # the counts bench.py reports as gpu_launches, per forward and backward
    w = WORKLOADS["text-32k"]
    assert B.kernel_launches(B.Params.from_workload(w)) == (8, 5)   # tcgen05 path, one sort pass
    assert B.kernel_launches(B.Params.from_workload(w.replace(sort_order="local"))) == (6, 5)
    assert B.kernel_launches(B.Params.from_workload(w.replace(sort_bits=12))) == (11, 5)
    # causal: token scan instead of |V| max + build; the key-major tcgen05
    # sparse backward + the dq cast (fp32: CUDA-core sparse backward + 3 casts)
    c = B.kernel_launches(B.Params.from_workload(w.replace(causal=True)))
    assert c == (1 + 3 + 1 + 1 + 1, 1 + 1 + 2 + 1)
    c = B.kernel_launches(B.Params.from_workload(w.replace(causal=True, dtype="f32")))
    assert c == (1 + 3 + 1 + 1 + 1, 1 + 1 + 4 + 1)
    # three hash rounds: every round's sort codes from the one hash GEMM, three
    # sorts, the inverse orders, the keys' earlier-round ranks, one
    # streamed-window pass per round and their combine; backward: one key-major pass per round + 3 casts (fp32: a second
    # hash kernel for the other rounds' codes and CUDA-core attention both ways)
    r = B.kernel_launches(B.Params.from_workload(w.replace(hash_rounds=3)))
    assert r == (1 + 3 * 3 + 1 + 2 + (1 + 3 + 1) + 1, 1 + 2 + (3 + 3) + 1)
    r = B.kernel_launches(B.Params.from_workload(w.replace(hash_rounds=3, dtype="f32")))
    assert r == (1 + 1 + 3 * 3 + 1 + 2 + 1 + 1, 1 + 2 + 1 + 3 + 1)


def test_path_flags():
    # the kernel families each workload takes (what the bench line and the
    # parity tests rely on)
    f = {n: B.path_flags(B.Params.from_workload(w)) for n, w in WORKLOADS.items()}
    main = ("tc_hash", "tc_attn", "slab_fwd", "slab_bwd")
    for n in ("text-32k", "vision-16k", "iid-4k"):
        assert all(f[n][k] for k in main) and not f[n]["tc_win"]
    # 10-bit RACE codes: the tables do not fit a shared-memory slab; d = 128
    # and 256-key chunks: the streamed-window forward
    assert f["needle-256k"]["tc_hash"] and f["needle-256k"]["tc_attn"]
    assert not f["needle-256k"]["slab_fwd"] and not f["needle-256k"]["slab_bwd"]
    assert f["needle-256k"]["tc_win"]
    # other lookbacks: the streamed-window forward and the key-major tcgen05
    # backward (not the persistent backward, which holds two query blocks)
    for lb in (0, 2, 5):
        g = B.path_flags(B.Params.from_workload(WORKLOADS["text-32k"].replace(lookback=lb)))
        assert g["tc_win"] and g["tc_attn"] and not g["slab_bwd"]
    assert not any(f["tiny-fp32"].values())
    w = WORKLOADS["text-32k"]
    assert not B.path_flags(B.Params.from_workload(w.replace(causal=True)))["slab_fwd"]
    assert not B.path_flags(B.Params.from_workload(w.replace(hash_rounds=2)))["slab_bwd"]
    assert B.path_flags(B.Params.from_workload(w.replace(hash_rounds=2)))["slab_fwd"]
    assert B.path_flags(B.Params.make(1, 1, 256, 64, "bf16", 4, 64, 8, 6)) == {
        "tc_hash": True, "tc_attn": True, "slab_fwd": False, "slab_bwd": False, "tc_win": False}
    # fp32 and ragged lengths keep the CUDA-core attention; causal and several
    # hash rounds take the streamed-window forward and the key-major backward
    w = WORKLOADS["text-32k"]
    for x in (w.replace(dtype="f32"), w.replace(N=32768 + 64, chunk=64)):
        assert not B.path_flags(B.Params.from_workload(x))["tc_win"]
    r = B.path_flags(B.Params.from_workload(w.replace(hash_rounds=2)))
    assert r["tc_win"] and r["tc_attn"] and not r["slab_bwd"]
    c = B.path_flags(B.Params.from_workload(w.replace(causal=True)))
    assert c["tc_win"] and c["tc_attn"] and not c["slab_fwd"] and not c["slab_bwd"]


def test_binding_argument_counts_match_the_header():
    # every bound entry point takes as many arguments as its declaration
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    lib = B.lib()
    for name in B.EXPORTS:
        m = re.search(r"\b" + name + r"\s*\(([^)]*)\)\s*;", text)
        assert m, name
        params = [x for x in m.group(1).split(",") if x.strip() and x.strip() != "void"]
        argtypes = getattr(lib, name).argtypes
        assert argtypes is not None and len(argtypes) == len(params), \
            f"{name}: {len(argtypes or [])} bound, {len(params)} declared"
