"""Plain fp64 CPU oracle for the ELSAA attention operator.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute anything in this package: only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.
It shares no code with the CUDA path (no kernels, headers, helpers or
constants): it receives the same seeded inputs and nothing else.

Every function here is written from the ELSAA pages
("ELSAA: Efficient Low-Rank and Sparse Attention Approximation for Training
Transformers" and "Two Efficient Attentions, One Denominator Problem") in the
order the method takes its steps, with library primitives (matmul, stable
argsort, bincount, index_add, logsumexp) as the only building blocks.

Parity status of each function (what pins it, see ``tests/test_oracle.py``):
  simhash_codes        pinned: brute-force sign loop, scale/negation invariants,
                       angular collision statistics
  stable_sort_perm     pinned: pure-Python sort by (code, index), permutation
                       and ordering properties
  gray_rank / sort_keys
                       pinned: inverts the enumerated reflected Gray code,
                       one-bit steps between neighbouring buckets, brute-force
                       stable sort by Gray position; local order = token order
                       with a banded dense mask
  sparse_branch        pinned: one chunk == dense softmax attention, masked dense
                       softmax over the rank mask (lookback 0 to 3 chunks),
                       one-hot value support test, closed form for Q = 0
  race_build / race_query
                       pinned: per-table sums, K_r = 0 closed form, collision
                       count matrix brute force
  sparse_branch_rounds / round_perms
                       pinned: one round equals sparse_branch, a repeated round
                       adds nothing (keys counted once), pure-Python union of
                       windows, mass never below any single round's
  race_query_causal    pinned: pure-Python loop over (query, table, key j <= i),
                       last token equals the full read-out, causal dense
                       identities through forward_head
  gates / fuse         pinned: hand-worked learned gates (distinct weight rows,
                       nonzero biases, q != 0, tokens out of sorted order),
                       lambda = 0 ablation (m == 1), single-branch gate
                       settings, Z_race = 0, closed form for Q = 0
  forward_head         pinned through the pieces above and the Q = 0 closed form
  grads_head           pinned: finite differences (gradcheck) of forward_head,
                       RACE branch carries no dq/dk
  interaction_count    parity unpinned (the pages lost the complexity formula;
                       only its 32K example survives)
"""

from .elsaa_oracle import (  # noqa: F401
    simhash_projections,
    simhash_codes,
    stable_sort_perm,
    gray_rank,
    sort_keys,
    SORT_ORDERS,
    chunk_window,
    sparse_branch,
    sparse_branch_rounds,
    round_perms,
    race_build,
    race_query,
    race_query_causal,
    gates,
    fuse,
    forward_head,
    grads_head,
    forward_batch,
    interaction_count,
    NEAR_ZERO,
)
