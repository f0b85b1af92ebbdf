"""Pins of the fp64 oracle against facts fixed by the pages and by mathematics,
independent of the oracle's own code paths (CPU only)."""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

F64 = torch.float64
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=F64)


# --------------------------------------------------------------------------- hash

def test_hash_matches_python_sign_loop():
    x = rnd((13, 5), 1)
    planes = rnd((7, 5), 2)
    got = O.simhash_codes(O.simhash_projections(x, planes))
    for i in range(13):
        code = 0
        for j in range(7):
            s = 0.0
            for t in range(5):
                s += float(x[i, t]) * float(planes[j, t])
            if s > 0:
                code += 2 ** j
        assert int(got[i]) == code


def test_hash_bit_order_and_zero_rule():
    planes = torch.tensor([[1.0, 0.0], [0.0, 1.0]], dtype=F64)
    x = torch.tensor([[1.0, 0.0], [0.0, 1.0], [-1.0, 2.0], [0.0, 0.0], [3.0, 3.0]], dtype=F64)
    # plane 0 gives bit 0 (weight 1), plane 1 bit 1 (weight 2); exactly 0 -> bit 0
    assert O.simhash_codes(O.simhash_projections(x, planes)).tolist() == [1, 2, 2, 0, 3]


def test_hash_scale_and_negation_invariance():
    x = rnd((200, 16), 3)
    planes = rnd((10, 16), 4)
    c = O.simhash_codes(O.simhash_projections(x, planes))
    c_scaled = O.simhash_codes(O.simhash_projections(3.7 * x, planes))
    c_neg = O.simhash_codes(O.simhash_projections(-x, planes))
    assert torch.equal(c, c_scaled)
    assert torch.equal(c_neg, (2 ** 10 - 1) - c)


def test_hash_collision_rate_is_angular():
    # SimHash: P[h(x) = h(y)] = (1 - theta/pi)^K for K independent hyperplanes
    d, K, trials = 8, 3, 20000
    g = torch.Generator().manual_seed(5)
    x = torch.zeros(d, dtype=F64); x[0] = 1.0
    theta = 1.0
    y = torch.zeros(d, dtype=F64); y[0] = math.cos(theta); y[1] = math.sin(theta)
    planes = torch.randn(trials, K, d, generator=g, dtype=F64)
    cx = O.simhash_codes(torch.einsum("tkd,d->tk", planes, x))
    cy = O.simhash_codes(torch.einsum("tkd,d->tk", planes, y))
    rate = (cx == cy).double().mean().item()
    expect = (1 - theta / math.pi) ** K
    assert abs(rate - expect) < 4 * math.sqrt(expect * (1 - expect) / trials)


# --------------------------------------------------------------------------- sort

def test_sort_is_stable_by_code_then_index():
    g = torch.Generator().manual_seed(6)
    code = torch.randint(0, 5, (300,), generator=g)
    perm = O.stable_sort_perm(code)
    expect = sorted(range(300), key=lambda i: (int(code[i]), i))
    assert perm.tolist() == expect
    assert sorted(perm.tolist()) == list(range(300))
    c = code[perm]
    assert bool((c[1:] >= c[:-1]).all())


# --------------------------------------------------------------------------- sparse branch

def test_one_chunk_is_dense_softmax_attention():
    n, d = 48, 8
    q, k, v = rnd((n, d), 7), rnd((n, d), 8), rnd((n, d), 9)
    perm = torch.randperm(n, generator=torch.Generator().manual_seed(1))
    perm2 = torch.randperm(n, generator=torch.Generator().manual_seed(2))
    o, lse = O.sparse_branch(q, k, v, perm, perm2, n, 0.3)
    ref = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None], scale=0.3)[0]
    assert torch.allclose(o, ref, atol=1e-12, rtol=0)
    assert torch.allclose(lse, torch.logsumexp(0.3 * q @ k.T, dim=1), atol=1e-12, rtol=0)


def test_sparse_equals_masked_dense_softmax():
    n, d, c = 40, 6, 8
    q, k, v = rnd((n, d), 10), rnd((n, d), 11), rnd((n, d), 12)
    pq = torch.randperm(n, generator=torch.Generator().manual_seed(3))
    pk = torch.randperm(n, generator=torch.Generator().manual_seed(4))
    o, lse = O.sparse_branch(q, k, v, pq, pk, c, 0.5)
    rank_q = {int(t): r for r, t in enumerate(pq)}
    rank_k = {int(t): r for r, t in enumerate(pk)}
    mask = torch.zeros(n, n, dtype=torch.bool)
    for i in range(n):
        for j in range(n):
            cq, ck = rank_q[i] // c, rank_k[j] // c
            mask[i, j] = ck == cq or ck == cq - 1
    s = 0.5 * q @ k.T
    s = s.masked_fill(~mask, float("-inf"))
    assert torch.allclose(o, torch.softmax(s, 1) @ v, atol=1e-12, rtol=0)
    assert torch.allclose(lse, torch.logsumexp(s, 1), atol=1e-12, rtol=0)
    # chunk 0 sees only its own c keys, later chunks 2c
    counts = mask.sum(1)
    for i in range(n):
        assert int(counts[i]) == (c if rank_q[i] < c else 2 * c)


def test_one_hot_values_expose_the_window():
    n, c = 32, 8
    q, k = rnd((n, n), 13), rnd((n, n), 14)
    v = torch.eye(n, dtype=F64)
    pq = torch.arange(n).flip(0)
    pk = torch.randperm(n, generator=torch.Generator().manual_seed(5))
    w, _ = O.sparse_branch(q, k, v, pq, pk, c, 0.2)
    for i in range(n):
        r = int((pq == i).nonzero())
        lo, hi = O.chunk_window(r, c)
        keys = set(pk[lo:hi].tolist())
        for j in range(n):
            assert (w[i, j] > 0) == (j in keys)
        assert abs(float(w[i].sum()) - 1) < 1e-12


# --------------------------------------------------------------------------- RACE

def test_race_tables_conserve_counts_and_values():
    n, d, L, kr = 100, 5, 6, 3
    g = torch.Generator().manual_seed(15)
    rk = torch.randint(0, 2 ** kr, (n, L), generator=g)
    v = rnd((n, d), 16)
    C, T = O.race_build(rk, v, 2 ** kr)
    assert C.shape == (L, 2 ** kr) and T.shape == (L, 2 ** kr, d)
    assert (C.sum(1) == n).all()
    assert torch.allclose(T.sum(1), v.sum(0).expand(L, d), atol=1e-12)


def test_race_with_zero_bits_is_global_mean():
    n, d, L = 64, 4, 5
    v = rnd((n, d), 17)
    rk = torch.zeros(n, L, dtype=torch.int64)
    C, T = O.race_build(rk, v, 1)
    ctot, o_race, z_race = O.race_query(torch.zeros(n, L, dtype=torch.int64), C, T)
    assert (ctot == n * L).all()
    assert torch.allclose(o_race, v.mean(0).expand(n, d), atol=1e-12)
    assert torch.allclose(z_race, torch.full((n,), float(n), dtype=F64))


def test_race_matches_collision_count_matrix():
    n, d, L, kr = 50, 3, 4, 2
    g = torch.Generator().manual_seed(18)
    rq = torch.randint(0, 2 ** kr, (n, L), generator=g)
    rk = torch.randint(0, 2 ** kr, (n, L), generator=g)
    v = rnd((n, d), 19)
    C, T = O.race_build(rk, v, 2 ** kr)
    ctot, o_race, z_race = O.race_query(rq, C, T)
    cnt = np.zeros((n, n))
    for i in range(n):
        for j in range(n):
            cnt[i, j] = sum(int(rq[i, l] == rk[j, l]) for l in range(L))
    den = cnt.sum(1)
    num = cnt @ v.numpy()
    for i in range(n):
        assert int(ctot[i]) == den[i]
        assert abs(float(z_race[i]) - den[i] / L) < 1e-12
        if den[i] > 0:
            assert np.allclose(o_race[i].numpy(), num[i] / den[i], atol=1e-12)
        else:
            assert torch.all(o_race[i] == 0)


# --------------------------------------------------------------------------- fusion and gates

def _unit(n=64, d=8, c=16, bs=2, L=3, kr=3, seed=20):
    q, k, v = rnd((n, d), seed), rnd((n, d), seed + 1), rnd((n, d), seed + 2)
    rs, rr = rnd((bs, d), seed + 3), rnd((L, kr, d), seed + 4)
    gw, gb = 0.3 * rnd((2, d), seed + 5), rnd((2,), seed + 6)
    return q, k, v, rs, rr, gw, gb


def test_lambda_zero_is_the_uncorrected_hybrid():
    q, k, v, rs, rr, gw, gb = _unit()
    out = O.forward_head(q, k, v, rs, rr, 16, None, gw, gb, lam=0.0)
    assert torch.equal(out["m"], torch.ones_like(out["m"]))
    y0 = out["g_s"][:, None] * out["o_sp"] + out["g_r"][:, None] * out["o_race"]
    assert torch.allclose(out["y"], y0, atol=1e-14)


def test_single_branch_gate_settings():
    q, k, v, rs, rr, _, _ = _unit()
    sp = O.forward_head(q, k, v, rs, rr, 16, None, lam=0.0, fixed_gates=(1.0, 0.0))
    assert torch.allclose(sp["y"], sp["o_sp"], atol=1e-14)
    rc = O.forward_head(q, k, v, rs, rr, 16, None, lam=2.0, fixed_gates=(0.0, 1.0))
    assert torch.allclose(rc["y"], rc["o_race"], atol=1e-14)
    both = O.forward_head(q, k, v, rs, rr, 16, None, lam=2.0, fixed_gates=(1.0, 0.0))
    assert torch.allclose(both["y"], both["m"][:, None] * both["o_sp"], atol=1e-14)
    assert bool((both["m"] < 1).all()) and bool((both["m"] > 0).all())


def test_empty_race_bucket_leaves_sparse_branch_unscaled():
    n, d, c = 32, 4, 8
    q, k, v = rnd((n, d), 30), rnd((n, d), 31), rnd((n, d), 32)
    rs = rnd((2, d), 33)
    rr = torch.zeros(1, 1, d, dtype=F64); rr[0, 0, 0] = 1.0
    q[:, 0] = q[:, 0].abs() + 0.1   # every query in bucket 1
    k[:, 0] = -k[:, 0].abs() - 0.1  # every key in bucket 0
    out = O.forward_head(q, k, v, rs, rr, c, None, lam=5.0, fixed_gates=(0.7, 0.4))
    assert (out["ctot"] == 0).all()
    assert torch.equal(out["m"], torch.ones(n, dtype=F64))
    assert torch.all(out["o_race"] == 0)
    assert torch.allclose(out["y"], 0.7 * out["o_sp"], atol=1e-14)


def test_hand_worked_four_token_example():
    """Every step of a 4-token, d = 2 example written out with scalars."""
    q = torch.tensor([[1.0, 1.0], [-1.0, 1.0], [0.5, -1.0], [-2.0, -1.0]], dtype=F64)
    k = torch.tensor([[1.0, 0.0], [-1.0, 1.0], [2.0, -1.0], [0.0, 1.0]], dtype=F64)
    v = torch.tensor([[1.0, 2.0], [3.0, -1.0], [0.0, 4.0], [-2.0, 1.0]], dtype=F64)
    rs = torch.tensor([[1.0, 0.0]], dtype=F64)          # sort bit = [x0 > 0]
    rr = torch.tensor([[[0.0, 1.0]]], dtype=F64)        # one table, bit = [x1 > 0]
    lam, gs, gr = 0.5, 0.8, 0.3
    out = O.forward_head(q, k, v, rs, rr, 2, None, lam=lam, fixed_gates=(gs, gr))
    # sort codes q: [1,0,1,0] -> order 1,3,0,2; k: [1,0,1,0] (k3 has x0 = 0 -> bit 0)
    assert out["perm_q"].tolist() == [1, 3, 0, 2]
    assert out["perm_k"].tolist() == [1, 3, 0, 2]
    sc = 1 / math.sqrt(2)
    dot = lambda a, b: a[0] * b[0] + a[1] * b[1]
    Q, K, V = q.tolist(), k.tolist(), v.tolist()
    # chunk 0 = queries {1, 3} see keys {1, 3}; chunk 1 = queries {0, 2} see all keys
    windows = {1: [1, 3], 3: [1, 3], 0: [1, 3, 0, 2], 2: [1, 3, 0, 2]}
    # RACE table: key bits [x1 > 0] = [0,1,0,1]: bucket 0 = {0, 2}, bucket 1 = {1, 3}
    buckets = {0: [0, 2], 1: [1, 3]}
    for i in range(4):
        e = [math.exp(sc * dot(Q[i], K[j])) for j in windows[i]]
        zsp = sum(e)
        osp = [sum(e[t] * V[j][c] for t, j in enumerate(windows[i])) / zsp for c in range(2)]
        b = 1 if Q[i][1] > 0 else 0
        keys = buckets[b]
        orace = [sum(V[j][c] for j in keys) / len(keys) for c in range(2)]
        zr = len(keys) / 1.0
        m = zsp / (zsp + lam * zr)
        y = [gs * m * osp[c] + gr * orace[c] for c in range(2)]
        assert abs(float(out["lse"][i]) - math.log(zsp)) < 1e-13
        assert abs(float(out["m"][i]) - m) < 1e-13
        assert int(out["ctot"][i]) == len(keys)
        for c in range(2):
            assert abs(float(out["o_sp"][i, c]) - osp[c]) < 1e-13
            assert abs(float(out["o_race"][i, c]) - orace[c]) < 1e-13
            assert abs(float(out["y"][i, c]) - y[c]) < 1e-13


def test_hand_worked_learned_gates():
    """The learned gates of the same 4-token example written out with scalars:
    g_s = sigmoid(w_s . q_i + b_s) from row 0 of the gate weights, g_r from row 1,
    q_i the query in token order (the sort puts the tokens in order 1, 3, 0, 2,
    so a gate taken at a sorted position would differ), no score scale on the
    gate logit (ELSAA overview: learned or fixed gates; "Two Efficient
    Attentions, One Denominator Problem", section "Two efficient branches can
    still be mis-scaled": independent token-wise gates)."""
    q = torch.tensor([[1.0, 1.0], [-1.0, 1.0], [0.5, -1.0], [-2.0, -1.0]], dtype=F64)
    k = torch.tensor([[1.0, 0.0], [-1.0, 1.0], [2.0, -1.0], [0.0, 1.0]], dtype=F64)
    v = torch.tensor([[1.0, 2.0], [3.0, -1.0], [0.0, 4.0], [-2.0, 1.0]], dtype=F64)
    rs = torch.tensor([[1.0, 0.0]], dtype=F64)
    rr = torch.tensor([[[0.0, 1.0]]], dtype=F64)
    gw = torch.tensor([[0.5, -0.25], [1.0, 0.75]], dtype=F64)   # row 0 sparse, row 1 RACE
    gb = torch.tensor([0.1, -0.2], dtype=F64)
    lam = 0.5
    out = O.forward_head(q, k, v, rs, rr, 2, None, gw, gb, lam=lam)
    assert out["perm_q"].tolist() == [1, 3, 0, 2]
    sig = lambda a: 1.0 / (1.0 + math.exp(-a))
    Q = q.tolist()
    # logits by hand: token 0: w_s.q = 0.5 - 0.25 = 0.25, w_r.q = 1.0 + 0.75 = 1.75
    a_s = [0.25, -0.75, 0.5, -0.75]
    a_r = [1.75, -0.25, -0.25, -2.75]
    for i in range(4):
        assert abs(0.5 * Q[i][0] - 0.25 * Q[i][1] - a_s[i]) < 1e-15
        assert abs(1.0 * Q[i][0] + 0.75 * Q[i][1] - a_r[i]) < 1e-15
        gs, gr = sig(a_s[i] + 0.1), sig(a_r[i] - 0.2)
        assert abs(float(out["g_s"][i]) - gs) < 1e-14
        assert abs(float(out["g_r"][i]) - gr) < 1e-14
        m = float(out["m"][i])
        for c in range(2):
            want = gs * m * float(out["o_sp"][i, c]) + gr * float(out["o_race"][i, c])
            assert abs(float(out["y"][i, c]) - want) < 1e-13
    # the two rows are not interchangeable on this example
    assert abs(float(out["g_s"][0]) - sig(1.75 + 0.1)) > 0.1
    # token 0 and token 2 swap places in the sorted order: their gates differ
    assert abs(float(out["g_s"][0]) - float(out["g_s"][2])) > 0.01


def test_zero_queries_closed_form():
    n, d, c, L, kr = 64, 6, 16, 5, 3
    k, v = rnd((n, d), 40), rnd((n, d), 41)
    q = torch.zeros(n, d, dtype=F64)
    rs, rr = rnd((3, d), 42), rnd((L, kr, d), 43)
    gw, gb = rnd((2, d), 44), torch.tensor([0.3, -1.2], dtype=F64)
    lam = 1.7
    out = O.forward_head(q, k, v, rs, rr, c, None, gw, gb, lam=lam)
    # q = 0: every projection is exactly 0, so every query code is 0, the query
    # order is the token order, every score is 0 and every gate is sigmoid(b).
    kcode = [sum(2 ** j for j in range(3) if float(k[t] @ rs[j]) > 0) for t in range(n)]
    korder = sorted(range(n), key=lambda t: (kcode[t], t))
    in0 = [sum(1 for t in range(n) if all(float(k[t] @ rr[l, j]) <= 0 for j in range(kr)))
           for l in range(L)]
    sum0 = [sum((v[t] for t in range(n) if all(float(k[t] @ rr[l, j]) <= 0 for j in range(kr))),
                torch.zeros(d, dtype=F64)) for l in range(L)]
    ctot = sum(in0)
    gs, gr = 1 / (1 + math.exp(-0.3)), 1 / (1 + math.exp(1.2))
    for i in range(n):
        lo, hi = max(0, (i // c - 1) * c), (i // c + 1) * c
        win = korder[lo:hi]
        osp = v[win].mean(0)
        orace = sum(sum0) / ctot if ctot else torch.zeros(d, dtype=F64)
        m = len(win) / (len(win) + lam * ctot / L)
        assert abs(float(out["lse"][i]) - math.log(len(win))) < 1e-12
        assert torch.allclose(out["o_sp"][i], osp, atol=1e-12)
        assert torch.allclose(out["y"][i], gs * m * osp + gr * orace, atol=1e-12)


# --------------------------------------------------------------------------- gradients

def test_gradients_match_finite_differences():
    n, d, c, L, kr = 12, 4, 4, 2, 2
    q, k, v, rs, rr, gw, gb = _unit(n, d, c, 2, L, kr, seed=50)
    first = O.forward_head(q, k, v, rs, rr, c, None, gw, gb, 0.7)
    codes = {x: first[x] for x in ("code_q", "code_k", "rcode_q", "rcode_k")}
    dy = rnd((n, d), 60)

    def f(q_, k_, v_, w_, b_, lam_):
        return O.forward_head(q_, k_, v_, rs, rr, c, None, w_, b_, lam_, codes=codes)["y"]

    args = tuple(t.clone().requires_grad_(True) for t in (q, k, v, gw, gb))
    lam = torch.tensor(0.7, dtype=F64, requires_grad=True)
    assert torch.autograd.gradcheck(f, args + (lam,), eps=1e-6, atol=1e-7)
    g = O.grads_head(q, k, v, rs, rr, c, dy, None, gw, gb, 0.7, codes=codes)
    loss = (f(*args, lam) * dy).sum()
    ref = torch.autograd.grad(loss, args + (lam,))
    for name, r in zip(("dq", "dk", "dv", "dgate_w", "dgate_b", "dlambda"), ref):
        assert torch.allclose(g[name], r, atol=1e-12)


def test_race_branch_carries_no_query_key_gradient():
    q, k, v, rs, rr, _, _ = _unit(32, 4, 8, 2, 3, 2, seed=70)
    dy = rnd((32, 4), 71)
    g = O.grads_head(q, k, v, rs, rr, 8, dy, None, lam=1.0, fixed_gates=(0.0, 1.0))
    assert torch.all(g["dq"] == 0) and torch.all(g["dk"] == 0)
    assert g["dv"].abs().sum() > 0


# --------------------------------------------------------------------------- the pages' one worked number

def test_interaction_count_example_order_of_magnitude():
    gold = json.load(open(os.path.join(GOLDEN, "interaction_count_32k.json")))
    n = gold["sequence_length"]
    assert n * n == gold["dense_pairwise_interactions"]
    # With chunk 128 and 64 tables every query scores about 2c keys and reads
    # L buckets: 2*128 + 64 = 320 per query, the example's 1.024e7 / 32000.
    cnt = O.interaction_count(32768, 128, 64)
    per_query = cnt["total"] / 32768
    assert abs(per_query - gold["elsaa_interactions"] / n) < 1.0


def test_zero_race_bits_through_forward_head():
    # K_r = 0: one bucket per table, every key collides with every query
    q, k, v, rs, _, gw, gb = _unit(32, 4, 8, 2, 3, 2, seed=80)
    rr = torch.zeros(3, 0, 4, dtype=F64)
    out = O.forward_head(q, k, v, rs, rr, 8, None, gw, gb, lam=1.0)
    assert (out["ctot"] == 3 * 32).all()
    assert torch.allclose(out["o_race"], v.mean(0).expand(32, 4), atol=1e-12)


# ---------------------------------------------------------------------------
# Sort-LSH bucket orders: Gray sequence and local windows
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [1, 2, 3, 5, 8, 16])
def test_gray_rank_inverts_the_reflected_gray_code(bits):
    # the reflected binary Gray code of position i is i ^ (i >> 1); its
    # position must come back from the code
    n = 1 << bits
    pos = torch.arange(n, dtype=torch.int64) if bits <= 12 else torch.randint(0, n, (4096,))
    codes = pos ^ (pos >> 1)
    assert torch.equal(O.gray_rank(codes), pos)


def test_gray_order_neighbours_differ_in_one_bit():
    bits = 6
    codes = torch.randint(0, 1 << bits, (500,), generator=torch.Generator().manual_seed(7))
    perm = O.stable_sort_perm(O.sort_keys(codes, "gray"))
    distinct = []
    for t in perm.tolist():
        c = int(codes[t])
        if not distinct or distinct[-1] != c:
            distinct.append(c)
    assert len(distinct) == len(set(distinct))   # each bucket is one contiguous run
    full = list(range(1 << bits))
    seq = [i ^ (i >> 1) for i in full]          # the Gray sequence, enumerated
    where = {c: i for i, c in enumerate(seq)}
    assert [where[c] for c in distinct] == sorted(where[c] for c in distinct)
    for a, b in zip(distinct, distinct[1:]):
        if where[b] == where[a] + 1:
            assert bin(a ^ b).count("1") == 1


def test_gray_sort_is_stable_brute_force():
    codes = torch.randint(0, 8, (60,), generator=torch.Generator().manual_seed(8))
    seq = [i ^ (i >> 1) for i in range(8)]
    pos = {c: i for i, c in enumerate(seq)}
    expect = sorted(range(60), key=lambda t: (pos[int(codes[t])], t))
    assert O.stable_sort_perm(O.sort_keys(codes, "gray")).tolist() == expect


def test_local_order_is_token_order_and_a_banded_mask():
    n, d, c = 48, 5, 8
    codes = torch.randint(0, 16, (n,), generator=torch.Generator().manual_seed(9))
    perm = O.stable_sort_perm(O.sort_keys(codes, "local"))
    assert torch.equal(perm, torch.arange(n))
    q, k, v = rnd((n, d), 15), rnd((n, d), 16), rnd((n, d), 17)
    o, lse = O.sparse_branch(q, k, v, perm, perm, c, 0.4)
    i = torch.arange(n)
    ci, cj = (i // c)[:, None], (i // c)[None, :]
    mask = (cj == ci) | (cj == ci - 1)          # own chunk and the previous one, in token order
    s = (0.4 * q @ k.T).masked_fill(~mask, float("-inf"))
    assert torch.allclose(o, torch.softmax(s, 1) @ v, atol=1e-12, rtol=0)
    assert torch.allclose(lse, torch.logsumexp(s, 1), atol=1e-12, rtol=0)


def test_sort_order_reaches_the_operator():
    n, d, c = 64, 8, 16
    q, k, v = rnd((n, d), 18), rnd((n, d), 19), rnd((n, d), 20)
    rs = rnd((3, d), 21).float()
    rr = rnd((2, 3, d), 22).float()
    outs = {o: O.forward_head(q, k, v, rs, rr, c, None, lam=1.0, fixed_gates=(0.5, 0.5),
                              sort_order=o) for o in O.SORT_ORDERS}
    assert torch.equal(outs["local"]["perm_q"], torch.arange(n))
    assert torch.equal(outs["gray"]["perm_q"],
                       O.stable_sort_perm(O.gray_rank(outs["gray"]["code_q"])))
    # the RACE branch does not depend on the order
    for o in ("gray", "local"):
        assert torch.allclose(outs[o]["o_race"], outs["binary"]["o_race"], atol=0, rtol=0)
    with pytest.raises(ValueError):
        O.sort_keys(outs["binary"]["code_q"], "spiral")


@pytest.mark.parametrize("lookback", [0, 2, 3])
def test_lookback_window_equals_masked_dense_softmax(lookback):
    n, d, c = 48, 6, 8
    q, k, v = rnd((n, d), 23), rnd((n, d), 24), rnd((n, d), 25)
    pq = torch.randperm(n, generator=torch.Generator().manual_seed(26))
    pk = torch.randperm(n, generator=torch.Generator().manual_seed(27))
    o, lse = O.sparse_branch(q, k, v, pq, pk, c, 0.5, lookback)
    rank_q = {int(t): r for r, t in enumerate(pq)}
    rank_k = {int(t): r for r, t in enumerate(pk)}
    mask = torch.zeros(n, n, dtype=torch.bool)
    for i in range(n):
        for j in range(n):
            cq, ck = rank_q[i] // c, rank_k[j] // c
            mask[i, j] = cq - lookback <= ck <= cq
    s = (0.5 * q @ k.T).masked_fill(~mask, float("-inf"))
    assert torch.allclose(o, torch.softmax(s, 1) @ v, atol=1e-12, rtol=0)
    assert torch.allclose(lse, torch.logsumexp(s, 1), atol=1e-12, rtol=0)
    for i in range(n):   # chunk j sees min(j, lookback) + 1 chunks
        assert int(mask[i].sum()) == c * (min(rank_q[i] // c, lookback) + 1)


def test_lookback_zero_with_one_chunk_is_dense_attention():
    n, d = 24, 5
    q, k, v = rnd((n, d), 28), rnd((n, d), 29), rnd((n, d), 30)
    pq = torch.randperm(n, generator=torch.Generator().manual_seed(31))
    pk = torch.randperm(n, generator=torch.Generator().manual_seed(32))
    o, _ = O.sparse_branch(q, k, v, pq, pk, n, 0.7, 0)
    ref = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None], scale=0.7)[0]
    assert torch.allclose(o, ref, atol=1e-12, rtol=0)


# ---------------------------------------------------------------------------
# causal ELSAA (an extension: keys j <= i only, in both branches)
# ---------------------------------------------------------------------------

def test_causal_one_local_chunk_is_causal_dense_attention():
    n, d = 20, 6
    q, k, v = rnd((n, d), 80), rnd((n, d), 81), rnd((n, d), 82)
    perm = torch.arange(n)
    o, lse = O.sparse_branch(q, k, v, perm, perm, n, 0.6, 0, causal=True)
    ref = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None],
                                                           is_causal=True, scale=0.6)[0]
    assert torch.allclose(o, ref, atol=1e-12, rtol=0)
    s = (0.6 * q @ k.T).masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), float("-inf"))
    assert torch.allclose(lse, torch.logsumexp(s, 1), atol=1e-12, rtol=0)


def test_causal_window_brute_force_and_empty_windows():
    n, d, c = 32, 5, 8
    q, k, v = rnd((n, d), 83), rnd((n, d), 84), rnd((n, d), 85)
    pq = torch.randperm(n, generator=torch.Generator().manual_seed(86))
    pk = torch.arange(n).flip(0)   # late keys first: early queries find no earlier key
    o, lse = O.sparse_branch(q, k, v, pq, pk, c, 0.5, 1, causal=True)
    rank_q = {int(t): r for r, t in enumerate(pq)}
    rank_k = {int(t): r for r, t in enumerate(pk)}
    empty = 0
    for i in range(n):
        keys = [j for j in range(n)
                if rank_q[i] // c - 1 <= rank_k[j] // c <= rank_q[i] // c and j <= i]
        if not keys:
            empty += 1
            assert float(lse[i]) == float("-inf") and torch.all(o[i] == 0)
            continue
        s = torch.stack([0.5 * q[i] @ k[j] for j in keys])
        p = torch.softmax(s, 0)
        assert abs(float(lse[i]) - float(torch.logsumexp(s, 0))) < 1e-12
        assert torch.allclose(o[i], sum(p[t] * v[j] for t, j in enumerate(keys)), atol=1e-12)
    assert empty > 0
    # gradients stay finite through the empty windows
    qg, kg, vg = (t.clone().requires_grad_(True) for t in (q, k, v))
    og, lg = O.sparse_branch(qg, kg, vg, pq, pk, c, 0.5, 1, causal=True)
    (og.sum() + lg[torch.isfinite(lg)].sum()).backward()
    assert all(torch.isfinite(t.grad).all() for t in (qg, kg, vg))


def test_causal_race_brute_force():
    n, L, nb, d = 24, 3, 4, 3
    g = torch.Generator().manual_seed(87)
    rq = torch.randint(0, nb, (n, L), generator=g)
    rk = torch.randint(0, nb, (n, L), generator=g)
    v = rnd((n, d), 88)
    ctot, o_race, z_race = O.race_query_causal(rq, rk, v)
    for i in range(n):
        cnt, num = 0, torch.zeros(d, dtype=F64)
        for l in range(L):
            for j in range(i + 1):
                if int(rq[i, l]) == int(rk[j, l]):
                    cnt += 1
                    num += v[j]
        assert int(ctot[i]) == cnt
        assert abs(float(z_race[i]) - cnt / L) < 1e-15
        assert torch.allclose(o_race[i], num / cnt if cnt else num, atol=1e-12)
    # the last token sees every key: the full read-out
    counts, sums = O.race_build(rk, v, nb)
    c_full, o_full, _ = O.race_query(rq, counts, sums)
    assert int(ctot[-1]) == int(c_full[-1])
    assert torch.allclose(o_race[-1], o_full[-1], atol=1e-12)


def test_fusion_with_an_empty_causal_window():
    n, d = 3, 2
    o_sp = torch.zeros(n, d, dtype=F64)
    lse = torch.full((n,), float("-inf"), dtype=F64)
    o_race = rnd((n, d), 89)
    z_race = torch.tensor([2.0, 0.0, 1.0], dtype=F64)
    g_s, g_r = torch.full((n,), 0.4, dtype=F64), torch.full((n,), 0.7, dtype=F64)
    y, m = O.fuse(o_sp, lse, o_race, z_race, g_s, g_r, 1.0)
    assert m.tolist() == [0.0, 1.0, 0.0]   # Z_sp = 0: m = 0, or 1 where both masses vanish
    assert torch.allclose(y, 0.7 * o_race, atol=1e-15)


def test_causal_gradients_match_finite_differences():
    n, d, c, L, kr = 12, 4, 4, 2, 2
    q, k, v, rs, rr, gw, gb = _unit(n, d, c, 2, L, kr, seed=90)
    first = O.forward_head(q, k, v, rs, rr, c, None, gw, gb, 0.7, causal=True)
    codes = {x: first[x] for x in ("code_q", "code_k", "rcode_q", "rcode_k")}
    dy = rnd((n, d), 91)

    def f(q_, k_, v_, w_, b_, lam_):
        return O.forward_head(q_, k_, v_, rs, rr, c, None, w_, b_, lam_, codes=codes,
                              causal=True)["y"]

    args = tuple(t.clone().requires_grad_(True) for t in (q, k, v, gw, gb))
    lam = torch.tensor(0.7, dtype=F64, requires_grad=True)
    assert torch.autograd.gradcheck(f, args + (lam,), eps=1e-6, atol=1e-7)
    g = O.grads_head(q, k, v, rs, rr, c, dy, None, gw, gb, 0.7, codes=codes, causal=True)
    assert all(torch.isfinite(g[x]).all() for x in ("dq", "dk", "dv", "dlambda"))


# ---------------------------------------------------------------------------
# several hash rounds (an extension): union of the rounds' windows, keys once
# ---------------------------------------------------------------------------

def test_one_round_is_the_sparse_branch():
    n, d, c = 48, 6, 8
    q, k, v = rnd((n, d), 100), rnd((n, d), 101), rnd((n, d), 102)
    rs = rnd((1, 3, d), 103)
    pq, pk = O.round_perms(q, k, rs)
    o1, l1 = O.sparse_branch(q, k, v, pq[0], pk[0], c, 0.4)
    o2, l2 = O.sparse_branch_rounds(q, k, v, pq, pk, c, 0.4)
    assert torch.allclose(o1, o2, atol=1e-12, rtol=0)
    assert torch.allclose(l1, l2, atol=1e-12, rtol=0)


def test_a_repeated_round_adds_nothing_and_more_rounds_add_mass():
    n, d, c = 40, 5, 8
    q, k, v = rnd((n, d), 104), rnd((n, d), 105), rnd((n, d), 106)
    rs = rnd((3, 3, d), 107)
    pq, pk = O.round_perms(q, k, rs)
    o1, l1 = O.sparse_branch_rounds(q, k, v, pq[:1], pk[:1], c, 0.5)
    od, ld = O.sparse_branch_rounds(q, k, v, [pq[0], pq[0]], [pk[0], pk[0]], c, 0.5)
    assert torch.allclose(o1, od, atol=1e-12, rtol=0) and torch.allclose(l1, ld, atol=1e-12, rtol=0)
    o3, l3 = O.sparse_branch_rounds(q, k, v, pq, pk, c, 0.5)
    for t in range(3):
        _, lt = O.sparse_branch_rounds(q, k, v, pq[t:t + 1], pk[t:t + 1], c, 0.5)
        assert torch.all(l3 >= lt - 1e-12)


def test_rounds_union_brute_force():
    n, d, c = 24, 4, 4
    q, k, v = rnd((n, d), 108), rnd((n, d), 109), rnd((n, d), 110)
    g = torch.Generator().manual_seed(111)
    pq = [torch.randperm(n, generator=g) for _ in range(2)]
    pk = [torch.randperm(n, generator=g) for _ in range(2)]
    o, lse = O.sparse_branch_rounds(q, k, v, pq, pk, c, 0.6)
    for i in range(n):
        keys = set()
        for t in range(2):
            ri = int((pq[t] == i).nonzero()) // c
            for j in range(n):
                rj = int((pk[t] == j).nonzero()) // c
                if ri - 1 <= rj <= ri:
                    keys.add(j)
        keys = sorted(keys)
        s = torch.stack([0.6 * q[i] @ k[j] for j in keys])
        p = torch.softmax(s, 0)
        assert abs(float(lse[i]) - float(torch.logsumexp(s, 0))) < 1e-12
        assert torch.allclose(o[i], sum(p[t] * v[j] for t, j in enumerate(keys)), atol=1e-12)


def test_rounds_through_forward_head():
    """forward_head with [R, b_s, d] hyperplanes: one round in 3-D form is the
    2-D one-round operator; a repeated round changes nothing; two distinct
    rounds give the union-window sparse branch, the same RACE branch and
    round 0's codes as the one-round call."""
    n, d, c, L, kr = 64, 6, 16, 3, 2
    q, k, v, rs, rr, gw, gb = _unit(n, d, c, 3, L, kr, seed=120)
    one = O.forward_head(q, k, v, rs, rr, c, None, gw, gb, 0.8)
    one3 = O.forward_head(q, k, v, rs[None], rr, c, None, gw, gb, 0.8)
    assert torch.equal(one["y"], one3["y"])
    rep = O.forward_head(q, k, v, torch.stack([rs, rs]), rr, c, None, gw, gb, 0.8)
    assert torch.allclose(rep["y"], one["y"], atol=1e-13, rtol=0)
    rs2 = torch.stack([rs, rnd(tuple(rs.shape), 121)])
    two = O.forward_head(q, k, v, rs2, rr, c, None, gw, gb, 0.8)
    assert torch.equal(two["code_q"], one["code_q"]) and torch.equal(two["round_code_q"][0],
                                                                     one["code_q"])
    assert torch.equal(two["o_race"], one["o_race"])
    pq, pk = O.round_perms(q, k, rs2)
    o, lse = O.sparse_branch_rounds(q.to(F64), k.to(F64), v.to(F64), pq, pk, c,
                                    1 / math.sqrt(d))
    assert torch.allclose(two["o_sp"], o, atol=1e-13, rtol=0)
    assert torch.all(two["lse"] >= one["lse"] - 1e-12) and bool((two["lse"] > one["lse"]).any())


def test_rounds_gradients_match_finite_differences():
    n, d, c, L, kr = 16, 4, 4, 2, 2
    q, k, v, rs, rr, gw, gb = _unit(n, d, c, 2, L, kr, seed=130)
    rs2 = torch.stack([rs, rnd(tuple(rs.shape), 131)])
    first = O.forward_head(q, k, v, rs2, rr, c, None, gw, gb, 0.7)
    codes = {x: first[x] for x in ("code_q", "code_k", "rcode_q", "rcode_k", "round_code_q",
                                   "round_code_k")}

    def f(q_, k_, v_, w_, b_, lam_):
        return O.forward_head(q_, k_, v_, rs2, rr, c, None, w_, b_, lam_, codes=codes)["y"]

    args = tuple(t.clone().requires_grad_(True) for t in (q, k, v, gw, gb))
    lam = torch.tensor(0.7, dtype=F64, requires_grad=True)
    assert torch.autograd.gradcheck(f, args + (lam,), eps=1e-6, atol=1e-7)
