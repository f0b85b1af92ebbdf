"""fp64 reference for the ELSAA attention operator (test infrastructure only).

ELSAA ("ELSAA: Efficient Low-Rank and Sparse Attention Approximation for
Training Transformers", overview) is the attention that follows the dense
Q/K/V projections.  It adds an exact sparse branch and a low-rank RACE branch,
rescales the sparse branch by its attention mass relative to the RACE mass and
mixes both through independent token-wise gates.

The pages lost their display formulas ("Two Efficient Attentions, One
Denominator Problem", section "Two efficient branches can still be
mis-scaled": the multiplier and the gated sum are missing).  The readings this
oracle takes where the text is silent are stated next to each step and, in
full, in the repository's design notes:

  * hashing is SimHash (sign of a projection on a random hyperplane), bit j of
    a code has weight 2**j, a projection of exactly 0 gives bit 0;
  * one shared set of hyperplanes for Q and K and for every (batch, head);
  * Sort-LSH orders Q and K separately by code, ties by token index; sorted
    query chunk j attends sorted key chunks j-1 and j (chunk 0: only its own),
    no wrap-around;
  * RACE: L tables of 2**K_r buckets, T[l][b] = sum of values, C[l][b] = count;
    O_race = sum_l T[l][h_l(q)] / sum_l C[l][h_l(q)] (0 when the count is 0),
    Z_race = sum_l C[l][h_l(q)] / L, each collision weighing exp(0) = 1;
  * m = Z_sp / (Z_sp + lambda * Z_race) with Z_sp = sum of exp(score) over the
    sparse window (unshifted), and y = g_s * m * O_sp + g_r * O_race;
  * gates g = sigmoid(w . q_i + b) per branch, or fixed constants;
  * score scale 1/sqrt(d) unless given.

All arithmetic is fp64 on the CPU.  Inputs are the exact values the device
sees (bf16 or fp32), upcast.
"""

from __future__ import annotations

import math
from typing import Dict, Optional

import numpy as np
import torch

F64 = torch.float64

# Projections with |x . r| below this are reported separately: their sign can
# legitimately differ between an fp64 dot product and an fp32-accumulated one.
NEAR_ZERO = 1e-5


# ---------------------------------------------------------------------------
# Step 1: SimHash codes
# ---------------------------------------------------------------------------

def simhash_projections(x: torch.Tensor, planes: torch.Tensor) -> torch.Tensor:
    """Projections x . r_j of every row of ``x`` [n, d] on every hyperplane
    ``planes`` [m, d], in fp64.  ELSAA overview: the sparse branch is selected
    by LSH; SimHash is the angular LSH whose edge model the page "Two
    Efficient Attentions, One Denominator Problem" (section "Full rank explains
    structural complementarity") relies on."""
    return x.to(F64) @ planes.to(F64).T


def simhash_codes(proj: torch.Tensor) -> torch.Tensor:
    """Integer codes from projections [n, m]: bit j = (proj[:, j] > 0), code =
    sum_j bit_j * 2**j.  A projection of exactly zero gives bit 0."""
    m = proj.shape[-1]
    bits = (proj > 0).to(torch.int64)
    weights = torch.tensor([1 << j for j in range(m)], dtype=torch.int64)
    return (bits * weights).sum(dim=-1)


# ---------------------------------------------------------------------------
# Step 2: Sort-LSH ordering
# ---------------------------------------------------------------------------

def stable_sort_perm(code: torch.Tensor) -> torch.Tensor:
    """perm[r] = token index at sorted rank r; stable (equal codes keep token
    order).  "The ablation isolates the actual contribution" names the
    Sort-LSH + RACE hybrid; sorting by hash code is what makes consecutive
    chunks hold similar tokens."""
    return torch.from_numpy(np.argsort(code.numpy(), kind="stable").astype(np.int64))


SORT_ORDERS = ("binary", "gray", "local")


def gray_rank(code: torch.Tensor) -> torch.Tensor:
    """Position of each code in the reflected binary Gray sequence, i.e. the
    b with b ^ (b >> 1) == code (prefix XOR of the code's bits from the top).
    Ordering buckets this way makes neighbouring buckets differ in one
    hyperplane; this is an extension of the pages' binary bucket order."""
    b = code.to(torch.int64).clone()
    shift = 1
    while shift < 32:
        b ^= b >> shift
        shift <<= 1
    return b


def sort_keys(code: torch.Tensor, order: str = "binary") -> torch.Tensor:
    """The key Sort-LSH sorts by.  binary: the code itself (the pages' Sort-LSH);
    gray: the code's Gray-sequence position; local: one key for every token,
    so the stable order is token order and chunks are local windows of
    consecutive tokens (the ELSAA overview lists local windows among the
    sparse patterns)."""
    if order == "binary":
        return code
    if order == "gray":
        return gray_rank(code)
    if order == "local":
        return torch.zeros_like(code)
    raise ValueError(f"unknown sort order {order!r}")


def chunk_window(rank: int, chunk: int, lookback: int = 1) -> tuple:
    """Sorted key ranks [lo, hi) seen by the query at sorted rank ``rank``:
    its own chunk and the previous one (chunk 0 only itself), no wrap-around.
    ``lookback`` previous chunks instead of one is an extension (0: the own
    chunk only); the pages' Sort-LSH is lookback = 1."""
    j = rank // chunk
    return max(0, (j - lookback) * chunk), (j + 1) * chunk


# ---------------------------------------------------------------------------
# Step 3: exact sparse branch
# ---------------------------------------------------------------------------

def sparse_branch(q, k, v, perm_q, perm_k, chunk: int, scale: float, lookback: int = 1,
                  causal: bool = False):
    """Exact softmax attention restricted to the Sort-LSH window ("Two
    Efficient Attentions, One Denominator Problem", section "Two efficient
    branches can still be mis-scaled": the sparse branch computes only the
    selected interactions, exactly).  Returns (O_sp [N, d], lse [N]) in token
    order; Z_sp = exp(lse) is the unshifted attention mass of the window.

    ``causal`` (an extension: the pages note that causal use was not
    evaluated) keeps only the keys of the window whose token index is at most
    the query's; a query with no such key gets O_sp = 0 and lse = -inf
    (Z_sp = 0)."""
    n = q.shape[0]
    qs, ks, vs = q[perm_q], k[perm_k], v[perm_k]
    outs, lses = [], []
    for j in range(n // chunk):
        lo, hi = chunk_window(j * chunk, chunk, lookback)
        s = scale * (qs[j * chunk:(j + 1) * chunk] @ ks[lo:hi].T)
        if not causal:
            lses.append(torch.logsumexp(s, dim=1))
            outs.append(torch.softmax(s, dim=1) @ vs[lo:hi])
            continue
        allowed = perm_k[lo:hi][None, :] <= perm_q[j * chunk:(j + 1) * chunk][:, None]
        has = allowed.any(dim=1)
        # rows without a key take finite stand-in scores so that no NaN
        # reaches the gradients; their results are replaced below
        s = torch.where(allowed | ~has[:, None], s, torch.full_like(s, float("-inf")))
        lse_j = torch.logsumexp(s, dim=1)
        o_j = torch.softmax(s, dim=1) @ vs[lo:hi]
        lses.append(torch.where(has, lse_j, torch.full_like(lse_j, float("-inf"))))
        outs.append(torch.where(has[:, None], o_j, torch.zeros_like(o_j)))
    o_sorted = torch.cat(outs, 0)
    lse_sorted = torch.cat(lses, 0)
    inv = torch.empty_like(perm_q)
    inv[perm_q] = torch.arange(n, dtype=perm_q.dtype)
    return o_sorted[inv], lse_sorted[inv]


def sparse_branch_rounds(q, k, v, perms_q, perms_k, chunk: int, scale: float,
                         lookback: int = 1, causal: bool = False):
    """Several hash rounds (an extension; the pages use one round): every
    round t sorts Q and K by its own codes, and a query attends the union of
    its Sort-LSH windows over the rounds, each key once, with exact softmax.
    perms_q / perms_k: one permutation per round.  One round is exactly
    sparse_branch.  Written as a dense N x N mask (test sizes only)."""
    n = q.shape[0]
    allowed = torch.zeros(n, n, dtype=torch.bool)
    for pq, pk in zip(perms_q, perms_k):
        rank_q = torch.empty_like(pq)
        rank_q[pq] = torch.arange(n, dtype=pq.dtype)
        rank_k = torch.empty_like(pk)
        rank_k[pk] = torch.arange(n, dtype=pk.dtype)
        cq, ck = (rank_q // chunk)[:, None], (rank_k // chunk)[None, :]
        allowed |= (ck <= cq) & (ck >= cq - lookback)
    if causal:
        allowed &= torch.arange(n)[None, :] <= torch.arange(n)[:, None]
    has = allowed.any(dim=1)
    s = scale * (q @ k.T)
    s = torch.where(allowed | ~has[:, None], s, torch.full_like(s, float("-inf")))
    lse = torch.logsumexp(s, dim=1)
    o = torch.softmax(s, dim=1) @ v
    return (torch.where(has[:, None], o, torch.zeros_like(o)),
            torch.where(has, lse, torch.full_like(lse, float("-inf"))))


def round_perms(q, k, r_sort_rounds, sort_order: str = "binary"):
    """Sort-LSH permutations of Q and K for each round's hyperplanes
    (r_sort_rounds: [R, b_s, d]); returns (perms_q, perms_k) lists."""
    perms_q, perms_k = [], []
    for planes in r_sort_rounds:
        cq = simhash_codes(simhash_projections(q.to(F64), planes))
        ck = simhash_codes(simhash_projections(k.to(F64), planes))
        perms_q.append(stable_sort_perm(sort_keys(cq, sort_order)))
        perms_k.append(stable_sort_perm(sort_keys(ck, sort_order)))
    return perms_q, perms_k


# ---------------------------------------------------------------------------
# Step 4: low-rank RACE branch
# ---------------------------------------------------------------------------

def race_build(rcode_k: torch.Tensor, v: torch.Tensor, nbuckets: int):
    """RACE tables from key codes [N, L] and values [N, d]: C[l][b] = number
    of keys with h_l(k) = b, T[l][b] = sum of their values ("Two Efficient
    Attentions, One Denominator Problem": the RACE branch compresses the
    interaction structure into hash-bucket summaries)."""
    L = rcode_k.shape[1]
    d = v.shape[1]
    counts = torch.stack([torch.bincount(rcode_k[:, l], minlength=nbuckets) for l in range(L)])
    sums = torch.stack([
        torch.zeros(nbuckets, d, dtype=F64).index_add(0, rcode_k[:, l], v) for l in range(L)
    ])
    return counts, sums


def race_query_causal(rcode_q: torch.Tensor, rcode_k: torch.Tensor, v: torch.Tensor):
    """Causal RACE read-out (an extension): query i reads, in every table, only
    the keys j <= i of its bucket: Ctot_i = sum_l #{j <= i : h_l(k_j) = h_l(q_i)},
    O_race_i = sum of those keys' values / Ctot_i (0 when Ctot_i = 0),
    Z_race_i = Ctot_i / L.  Written as the collision-count matrix restricted to
    j <= i, a block of queries at a time.  Returns (Ctot, O_race, Z_race)."""
    n, L = rcode_q.shape
    ctot = torch.zeros(n, dtype=torch.int64)
    num = torch.zeros(n, v.shape[1], dtype=F64)
    for a in range(0, n, 512):
        b = min(n, a + 512)
        cnt = torch.zeros(b - a, n, dtype=torch.int64)
        for l in range(L):
            cnt += (rcode_q[a:b, l][:, None] == rcode_k[:, l][None, :]).to(torch.int64)
        cnt *= (torch.arange(n)[None, :] <= torch.arange(a, b)[:, None]).to(torch.int64)
        ctot[a:b] = cnt.sum(dim=1)
        num[a:b] = cnt.to(F64) @ v
    safe = torch.where(ctot > 0, ctot, torch.ones_like(ctot)).to(F64)
    o_race = torch.where((ctot > 0)[:, None], num / safe[:, None], torch.zeros_like(num))
    return ctot, o_race, ctot.to(F64) / L


def race_query(rcode_q: torch.Tensor, counts: torch.Tensor, sums: torch.Tensor):
    """Each query reads its bucket in every table: Ctot = sum_l C[l][h_l(q)],
    O_race = sum_l T[l][h_l(q)] / Ctot (0 when Ctot = 0), Z_race = Ctot / L
    (the RACE estimate of the collision-kernel mass, each colliding key
    weighing exp(0) = 1).  Returns (Ctot [N] int64, O_race [N, d], Z_race [N])."""
    L = rcode_q.shape[1]
    ctot = sum(counts[l][rcode_q[:, l]] for l in range(L))
    num = sum(sums[l][rcode_q[:, l]] for l in range(L))
    safe = torch.where(ctot > 0, ctot, torch.ones_like(ctot)).to(F64)
    o_race = torch.where((ctot > 0)[:, None], num / safe[:, None], torch.zeros_like(num))
    z_race = ctot.to(F64) / L
    return ctot, o_race, z_race


# ---------------------------------------------------------------------------
# Steps 5-6: denominator-aware fusion and token-wise gates
# ---------------------------------------------------------------------------

def gates(q, gate_w, gate_b, fixed: Optional[tuple] = None):
    """Independent token-wise gates, learned or fixed (ELSAA overview):
    g_s = sigmoid(w_s . q_i + b_s), g_r = sigmoid(w_r . q_i + b_r)."""
    n = q.shape[0]
    if fixed is not None:
        return (torch.full((n,), float(fixed[0]), dtype=F64),
                torch.full((n,), float(fixed[1]), dtype=F64))
    a_s = q @ gate_w[0] + gate_b[0]
    a_r = q @ gate_w[1] + gate_b[1]
    return torch.sigmoid(a_s), torch.sigmoid(a_r)


def fuse(o_sp, lse, o_race, z_race, g_s, g_r, lam):
    """Denominator-aware fusion ("Two Efficient Attentions, One Denominator
    Problem", section "Two efficient branches can still be mis-scaled"): the
    sparse output is scaled by its mass relative to the RACE mass,
    m = Z_sp / (Z_sp + lambda * Z_race), then both branches are gated
    independently: y = g_s * m * O_sp + g_r * O_race.  With lambda = 0 the
    multiplier is one (the Sort_Lsh_RACE ablation)."""
    z_sp = torch.exp(lse)
    den = z_sp + lam * z_race
    # m = 1 where both masses vanish (only a causal window can have Z_sp = 0);
    # the safe denominator keeps NaN out of the unused branch's gradient
    safe = torch.where(den > 0, den, torch.ones_like(den))
    m = torch.where(den > 0, z_sp / safe, torch.ones_like(den))
    y = g_s[:, None] * m[:, None] * o_sp + g_r[:, None] * o_race
    return y, m


# ---------------------------------------------------------------------------
# One (batch, head) unit, forward and gradients
# ---------------------------------------------------------------------------

def _hash_all(q64, k64, r_sort, r_race):
    L, kr, d = r_race.shape
    pq_s = simhash_projections(q64, r_sort)
    pk_s = simhash_projections(k64, r_sort)
    planes = r_race.reshape(L * kr, d)
    pq_r = simhash_projections(q64, planes).reshape(q64.shape[0], L, kr)
    pk_r = simhash_projections(k64, planes).reshape(k64.shape[0], L, kr)
    return pq_s, pk_s, pq_r, pk_r


def forward_head(q, k, v, r_sort, r_race, chunk: int, scale: Optional[float] = None,
                 gate_w=None, gate_b=None, lam=1.0, fixed_gates: Optional[tuple] = None,
                 codes: Optional[Dict[str, torch.Tensor]] = None,
                 sort_order: str = "binary", lookback: int = 1,
                 causal: bool = False) -> Dict[str, torch.Tensor]:
    """The whole operator on one (batch, head) unit.

    q, k, v: [N, d] (any float dtype; upcast to fp64).  r_sort: [b_s, d] for
    one Sort-LSH hash round, or [R, b_s, d] for R rounds (several rounds are an
    extension: sparse_branch_rounds); r_race: [L, K_r, d].  ``codes`` may
    carry precomputed code_q / code_k / rcode_q / rcode_k (and round_code_q /
    round_code_k [R, N] for several rounds; used to re-run the float steps with
    another side's codes where a projection sits within NEAR_ZERO of zero, and
    to freeze the hash in gradient checks).  Returns every intermediate in
    token order."""
    q64, k64, v64 = q.to(F64), k.to(F64), v.to(F64)
    n, d = q64.shape
    L, kr, _ = r_race.shape
    rounds = r_sort.shape[0] if r_sort.dim() == 3 else 1
    r_sort0 = r_sort[0] if r_sort.dim() == 3 else r_sort
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out: Dict[str, torch.Tensor] = {}
    if codes is None:
        with torch.no_grad():
            pq_s, pk_s, pq_r, pk_r = _hash_all(q64.detach(), k64.detach(), r_sort0, r_race)
        code_q, code_k = simhash_codes(pq_s), simhash_codes(pk_s)
        rcode_q, rcode_k = simhash_codes(pq_r), simhash_codes(pk_r)
        near = [p.abs() < NEAR_ZERO for p in (pq_s, pk_s, pq_r, pk_r)]
        out["near_code_q"] = near[0].any(dim=-1)
        out["near_code_k"] = near[1].any(dim=-1)
        out["near_rcode_q"] = near[2].any(dim=-1)
        out["near_rcode_k"] = near[3].any(dim=-1)
        if rounds > 1:
            with torch.no_grad():
                proj_q = [simhash_projections(q64.detach(), r_sort[t]) for t in range(rounds)]
                proj_k = [simhash_projections(k64.detach(), r_sort[t]) for t in range(rounds)]
            round_code_q = torch.stack([simhash_codes(p) for p in proj_q])
            round_code_k = torch.stack([simhash_codes(p) for p in proj_k])
            out["near_round_code_q"] = torch.stack([(p.abs() < NEAR_ZERO).any(-1) for p in proj_q])
            out["near_round_code_k"] = torch.stack([(p.abs() < NEAR_ZERO).any(-1) for p in proj_k])
    else:
        code_q, code_k = codes["code_q"].to(torch.int64), codes["code_k"].to(torch.int64)
        rcode_q, rcode_k = codes["rcode_q"].to(torch.int64), codes["rcode_k"].to(torch.int64)
        if rounds > 1:
            round_code_q = codes["round_code_q"].to(torch.int64)
            round_code_k = codes["round_code_k"].to(torch.int64)
    perm_q = stable_sort_perm(sort_keys(code_q, sort_order))
    perm_k = stable_sort_perm(sort_keys(code_k, sort_order))
    if rounds == 1:
        o_sp, lse = sparse_branch(q64, k64, v64, perm_q, perm_k, chunk, scale, lookback, causal)
    else:
        perms_q = [stable_sort_perm(sort_keys(c, sort_order)) for c in round_code_q]
        perms_k = [stable_sort_perm(sort_keys(c, sort_order)) for c in round_code_k]
        o_sp, lse = sparse_branch_rounds(q64, k64, v64, perms_q, perms_k, chunk, scale,
                                         lookback, causal)
        out.update(round_code_q=round_code_q, round_code_k=round_code_k,
                   round_perm_q=torch.stack(perms_q), round_perm_k=torch.stack(perms_k))
    counts, sums = race_build(rcode_k, v64, 1 << kr)
    if causal:
        ctot, o_race, z_race = race_query_causal(rcode_q, rcode_k, v64)
    else:
        ctot, o_race, z_race = race_query(rcode_q, counts, sums)
    if fixed_gates is None:
        g_s, g_r = gates(q64, gate_w.to(F64), gate_b.to(F64))
    else:
        g_s, g_r = gates(q64, None, None, fixed=fixed_gates)
    y, m = fuse(o_sp, lse, o_race, z_race, g_s, g_r, lam)
    out.update(code_q=code_q, code_k=code_k, rcode_q=rcode_q, rcode_k=rcode_k,
               perm_q=perm_q, perm_k=perm_k, o_sp=o_sp, lse=lse, race_count=counts,
               race_sum=sums, ctot=ctot, o_race=o_race, z_race=z_race, g_s=g_s, g_r=g_r,
               m=m, y=y)
    return out


def grads_head(q, k, v, r_sort, r_race, chunk: int, dy, scale: Optional[float] = None,
               gate_w=None, gate_b=None, lam=1.0, fixed_gates: Optional[tuple] = None,
               codes: Optional[Dict[str, torch.Tensor]] = None,
               sort_order: str = "binary", lookback: int = 1,
               causal: bool = False) -> Dict[str, torch.Tensor]:
    """Gradients of sum(y * dy) with the hash codes held constant (codes are
    piecewise constant in q and k), by fp64 autograd through forward_head.
    The pages state that ELSAA is used in training ("ELSAA combines sparsity
    and low-rank methods...": the approximation acts at run time during
    training).  Returns dq, dk, dv [N, d], dgate_w [2, d], dgate_b [2],
    dlambda (scalar); gate grads are zero for fixed gates."""
    q64 = q.to(F64).detach().requires_grad_(True)
    k64 = k.to(F64).detach().requires_grad_(True)
    v64 = v.to(F64).detach().requires_grad_(True)
    lam64 = torch.tensor(float(lam), dtype=F64, requires_grad=True)
    leaves = [q64, k64, v64, lam64]
    gw = gb = None
    if fixed_gates is None:
        gw = gate_w.to(F64).detach().requires_grad_(True)
        gb = gate_b.to(F64).detach().requires_grad_(True)
        leaves += [gw, gb]
    if codes is None:
        first = forward_head(q, k, v, r_sort, r_race, chunk, scale, gate_w, gate_b, lam,
                             fixed_gates, sort_order=sort_order, lookback=lookback,
                             causal=causal)
        codes = {name: first[name] for name in ("code_q", "code_k", "rcode_q", "rcode_k",
                                                "round_code_q", "round_code_k") if name in first}
    out = forward_head(q64, k64, v64, r_sort, r_race, chunk, scale, gw, gb, lam64,
                       fixed_gates, codes=codes, sort_order=sort_order, lookback=lookback,
                       causal=causal)
    loss = (out["y"] * dy.to(F64)).sum()
    g = torch.autograd.grad(loss, leaves, allow_unused=True)
    res = {"dq": g[0], "dk": g[1], "dv": g[2], "dlambda": g[3]}
    d = q.shape[1]
    if fixed_gates is None:
        res["dgate_w"], res["dgate_b"] = g[4], g[5]
    else:
        res["dgate_w"] = torch.zeros(2, d, dtype=F64)
        res["dgate_b"] = torch.zeros(2, dtype=F64)
    res["y"] = out["y"].detach()
    return res


def forward_batch(q, k, v, r_sort, r_race, chunk: int, scale=None, gate_w=None,
                  gate_b=None, lam=1.0, fixed_gates=None, units=None, sort_order="binary",
                  lookback=1):
    """forward_head over (batch, head) units of [B, H, N, d] tensors; ``units``
    selects a subset of (b, h) pairs (default all).  Returns {(b, h): dict}."""
    B, H = q.shape[0], q.shape[1]
    if units is None:
        units = [(b, h) for b in range(B) for h in range(H)]
    return {(b, h): forward_head(q[b, h], k[b, h], v[b, h], r_sort, r_race, chunk, scale,
                                 gate_w, gate_b, lam, fixed_gates, sort_order=sort_order,
                                 lookback=lookback)
            for (b, h) in units}


def interaction_count(n: int, chunk: int, race_tables: int) -> Dict[str, int]:
    """Attention-or-bucket interactions of one unit: every query scores the
    keys of its window and reads one bucket per RACE table.  "Linear
    interactions are not yet production economics" states the count is
    linear in N and gives a 32K example; its formula is lost (parity
    unpinned), so this is the count the algorithm above performs."""
    window = sum(min((j + 1) * chunk, n) - max(0, (j - 1) * chunk) for j in range(n // chunk))
    return {"sparse": window * chunk, "race": n * race_tables,
            "total": window * chunk + n * race_tables, "dense": n * n}
