"""The allocation-free Sort-LSH entry point against the regular forward.

elsaa_sort_codes_noalloc is for callers that cannot give the library scratch
memory while they run: a serving process whose memory pool already owns all
device memory, or a host framework that forbids cudaMalloc/cudaFree (they
synchronise the device) inside a step.  Its radix-sort scratch lives in a
fixed array inside the library, shared by every call, so the permutations it
returns must equal the ones elsaa_forward saves on every call, not only on the
first.  This file is collected last so that a run stopping at the first
failure has already run every other test.
"""

import ctypes

import pytest
import torch

from sparse_rank_hybrid_simhash_b200 import binding as B
from sparse_rank_hybrid_simhash_b200.workloads import WORKLOADS, make_inputs, small

pytestmark = pytest.mark.gpu

CASES = {
    "text-32k-small": small(WORKLOADS["text-32k"], B=1, H=2, N=1024),
    "two-radix-passes": WORKLOADS["iid-4k"].replace(B=1, H=2, N=1024, sort_bits=12),
    "needle-small": small(WORKLOADS["needle-256k"], B=1, H=2, N=2048),
    # Gray order transforms the key where the radix sort reads it; 12 bits
    # take two passes, so both the histograms and the intermediate order sit
    # in the library's scratch
    "gray-two-passes": WORKLOADS["iid-4k"].replace(B=1, H=2, N=1024, sort_bits=12,
                                                   sort_order="gray"),
    # local order writes token order and touches no scratch
    "local-order": WORKLOADS["iid-4k"].replace(B=1, H=2, N=1024, sort_order="local"),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_sort_matches_forward_permutations(cuda_device, name):
    w = CASES[name]
    p = B.Params.from_workload(w)
    d = {k: t.to(cuda_device) for k, t in make_inputs(w, with_dy=False).items()}
    saved = B.alloc_saved(p, cuda_device)
    ws = B.alloc_workspace(p, cuda_device)
    B.forward(p, d["q"], d["k"], d["v"], d["r_sort"], d["r_race"], d["gate_w"], d["gate_b"],
              d["lam"], saved=saved, ws=ws)
    B.check(ws)
    views = B.saved_views(p, saved)
    n = w.B * w.H * w.N
    # the query codes followed by the key codes, as one contiguous [2, B, H, N]
    codes = torch.cat([views["code_q"].reshape(-1), views["code_k"].reshape(-1)])
    expect = torch.cat([views["perm_q"].reshape(-1), views["perm_k"].reshape(-1)])
    for _ in range(2):                 # the second call sees the first call's scratch
        perm = torch.full((2 * n,), -1, dtype=torch.int32, device=cuda_device)
        B.sort_codes_noalloc(p, codes, perm)
        torch.cuda.synchronize()
        assert torch.equal(perm, expect)


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_device):
    # 12-bit codes need a second radix pass and 2 B H N ints of scratch: 8 MiB here
    p = B.Params.make(1, 1, 1 << 20, 64, "bf16", 12, 128, 4, 4)
    codes = torch.zeros(2 << 20, dtype=torch.int16, device=cuda_device)
    perm = torch.empty(2 << 20, dtype=torch.int32, device=cuda_device)
    status = B.lib().elsaa_sort_codes_noalloc(ctypes.byref(p), ctypes.c_void_p(codes.data_ptr()),
                                             ctypes.c_void_p(perm.data_ptr()),
                                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert status == 3   # ELSAA_ERR_WORKSPACE: more scratch than the built-in array holds
