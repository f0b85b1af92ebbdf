"""Seeded synthetic workloads for the ELSAA operator.

This module only draws random numbers and shapes them; it holds none of the
operator's arithmetic, so both the CUDA path and the CPU oracle may take their
inputs from it.  Every tensor is drawn in fp32 with ``numpy.random.default_rng``
and then rounded once to the workload's dtype; both sides consume exactly the
rounded values.

Workloads (shapes and value structure of the ELSAA evaluation, see "Two
Efficient Attentions, One Denominator Problem": 16K-token vision tasks, 32K
text classification, Needle-in-a-Haystack up to long lengths; no dataset is
available, so each is a synthetic stand-in of the same shape):

  tiny-fp32     B1 H1 N256 d32 fp32, iid N(0,1), 3-bit Sort-LSH, chunk 32,
                RACE 4 x 3-bit, fixed gates 0.5/0.5, lambda 1   (forward)
  iid-4k        B4 H8 N4096 d64 bf16, iid N(0,1), 4-bit, chunk 64,
                RACE 16 x 6-bit, learned gates w ~ N(0, 0.02^2), b = 0,
                lambda 1, dy ~ N(0,1)                          (fwd + bwd)
  vision-16k    B8 H8 N16384 d64 bf16, Q/K from a mixture of 64 Gaussian
                centres (norm 3, within std 0.5), V iid; 6-bit, chunk 128,
                RACE 32 x 8-bit, learned gates, learnable lambda (fwd + bwd)
  text-32k      B2 H12 N32768 d64 bf16, Q/K iid N(0,1) plus a Zipf(1.1)
                weighted prototype (512 per head), V iid; 7-bit, chunk 128,
                RACE 32 x 8-bit, learned gates                  (fwd + bwd)
  needle-256k   B1 H8 N262144 d128 bf16, iid with one planted key equal to
                4x a chosen query, 8-bit, chunk 256, RACE 64 x 10-bit (forward)
"""

from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str            # "bf16" or "f32"
    sort_bits: int
    chunk: int
    race_tables: int
    race_bits: int
    gate_fixed: bool
    gate_s: float = 0.5
    gate_r: float = 0.5
    gate_std: float = 0.02
    lam: float = 1.0
    backward: bool = True
    seed: int = 0
    dist: str = "iid"      # iid | clusters | zipf | needle
    sort_order: str = "binary"   # binary | gray | local (Sort-LSH bucket order)
    lookback: int = 1            # previous sorted chunks a query chunk attends
    causal: bool = False         # keys j <= i only
    hash_rounds: int = 1         # Sort-LSH hash rounds (each with its own hyperplanes)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def tokens(self) -> int:
        return self.B * self.N

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    "tiny-fp32": Workload("tiny-fp32", 1, 1, 256, 32, "f32", 3, 32, 4, 3, True,
                          0.5, 0.5, backward=False, seed=0, dist="iid"),
    "iid-4k": Workload("iid-4k", 4, 8, 4096, 64, "bf16", 4, 64, 16, 6, False,
                       seed=1, dist="iid"),
    "vision-16k": Workload("vision-16k", 8, 8, 16384, 64, "bf16", 6, 128, 32, 8, False,
                           seed=2, dist="clusters"),
    "text-32k": Workload("text-32k", 2, 12, 32768, 64, "bf16", 7, 128, 32, 8, False,
                         seed=3, dist="zipf"),
    "needle-256k": Workload("needle-256k", 1, 8, 262144, 128, "bf16", 8, 256, 64, 10, False,
                            backward=False, seed=4, dist="needle"),
}


def _normal(rng, shape):
    return rng.standard_normal(size=shape, dtype=np.float32)


def _qk_clusters(rng, B, H, N, d, centres=64, norm=3.0, std=0.5):
    q = np.empty((B, H, N, d), np.float32)
    k = np.empty((B, H, N, d), np.float32)
    for b in range(B):
        for h in range(H):
            c = _normal(rng, (centres, d))
            c *= norm / np.linalg.norm(c, axis=1, keepdims=True)
            uq = rng.integers(0, centres, size=N)
            uk = rng.integers(0, centres, size=N)
            q[b, h] = c[uq] + std * _normal(rng, (N, d))
            k[b, h] = c[uk] + std * _normal(rng, (N, d))
    return q, k


def _qk_zipf(rng, B, H, N, d, prototypes=512, s=1.1):
    p = np.arange(1, prototypes + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(p / p.sum())
    q = _normal(rng, (B, H, N, d))
    k = _normal(rng, (B, H, N, d))
    for b in range(B):
        for h in range(H):
            proto = _normal(rng, (prototypes, d))
            zq = np.minimum(np.searchsorted(cdf, rng.random(N)), prototypes - 1)
            zk = np.minimum(np.searchsorted(cdf, rng.random(N)), prototypes - 1)
            q[b, h] += proto[zq]
            k[b, h] += proto[zk]
    return q, k


def make_inputs(w: Workload, seed: Optional[int] = None, with_dy: Optional[bool] = None,
                device="cpu") -> Dict[str, torch.Tensor]:
    """Draw every input of one workload.  Returns torch tensors:
    q, k, v [B, H, N, d] and r_sort [b_s, d] (one hash round; [R, b_s, d] for
    R rounds, round 0 the same draw as for one round), r_race [L, K_r, d] in the
    workload dtype; gate_w [2, d], gate_b [2], lam [1] in fp32; dy (same shape
    and dtype as q) when the workload has a backward; for the needle workload
    also needle_key [B, H] and needle_query [B, H] (token indices)."""
    rng = np.random.default_rng(w.seed if seed is None else seed)
    B, H, N, d = w.B, w.H, w.N, w.d
    if w.dist == "clusters":
        q, k = _qk_clusters(rng, B, H, N, d)
    elif w.dist == "zipf":
        q, k = _qk_zipf(rng, B, H, N, d)
    else:
        q = _normal(rng, (B, H, N, d))
        k = _normal(rng, (B, H, N, d))
    v = _normal(rng, (B, H, N, d))
    extra = {}
    if w.dist == "needle":
        pk = rng.integers(0, N, size=(B, H))
        pq = rng.integers(0, N, size=(B, H))
        for b in range(B):
            for h in range(H):
                k[b, h, pk[b, h]] = 4.0 * q[b, h, pq[b, h]]
        extra["needle_key"] = torch.from_numpy(pk.astype(np.int64))
        extra["needle_query"] = torch.from_numpy(pq.astype(np.int64))
    r_sort = _normal(rng, (w.sort_bits, d))
    r_race = _normal(rng, (w.race_tables, w.race_bits, d))
    gate_w = (w.gate_std * _normal(rng, (2, d))).astype(np.float32)
    gate_b = np.zeros(2, np.float32)
    lam = np.array([w.lam], np.float32)
    dt = w.torch_dtype
    out = {
        "q": torch.from_numpy(q).to(dt), "k": torch.from_numpy(k).to(dt),
        "v": torch.from_numpy(v).to(dt),
        "r_sort": torch.from_numpy(r_sort).to(dt), "r_race": torch.from_numpy(r_race).to(dt),
        "gate_w": torch.from_numpy(gate_w), "gate_b": torch.from_numpy(gate_b),
        "lam": torch.from_numpy(lam),
    }
    if with_dy if with_dy is not None else w.backward:
        out["dy"] = torch.from_numpy(_normal(rng, (B, H, N, d))).to(dt)
    out.update(extra)
    if w.hash_rounds > 1:
        # the other rounds' hyperplanes are drawn last, so every other input
        # keeps its one-round values
        more = _normal(rng, (w.hash_rounds - 1, w.sort_bits, d))
        out["r_sort"] = torch.cat([out["r_sort"][None], torch.from_numpy(more).to(dt)], 0)
    if device != "cpu":
        out = {kk: t.to(device) for kk, t in out.items()}
    return out


def small(w: Workload, B=1, H=2, N=None) -> Workload:
    """The same workload (dtype, bits, chunk, tables, value structure) at a size
    the oracle finishes in seconds: N spans several chunks and query tiles."""
    n = N if N is not None else max(4 * w.chunk, 1024)
    return w.replace(name=w.name + "-small", B=B, H=H, N=n)
