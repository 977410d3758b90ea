"""Pins of the oracle's partition importance and importance plan ("DiTango",
error model and selection strategy) against facts outside the oracle: the
softmax mass of each key set by brute force, the weights summing to one, and
a second statement of the selection rule."""

import math

import numpy as np
import pytest

import oracle as orc
from partitioned_attention_state_b200 import workloads as wl


def run_anchor(H, S, D, P, group, seed):
    q, k, v = wl.InputStream(H, S, D, sigma=0.05, seed=seed).next_step()
    cache = orc.StateCache()
    plan, _, st = orc.build_plan(orc.MODE_ALL_COMPUTE, H, S, D, P, step=1, group=group)
    O, L, _ = orc.partition_step(q, k, v, plan, S, P, cache, group=group)
    Lmap = {(h, r): float(L[h, r]) for h in range(H) for r in range(S)}
    return (q, k, v), cache, Lmap, plan.shape[1], st


@pytest.mark.parametrize("S,P,g", [(60, 3, 0), (130, 4, 0), (200, 5, 2), (140, 4, 1)])
def test_importance_is_softmax_mass_of_each_key_set(S, P, g):
    """exp(LSE_k - LSE) of a row is the share of its softmax mass that falls
    on key set k: brute force with scalar loops over the full row."""
    H, D = 1, 4
    (q, k, v), cache, L, nseg, _ = run_anchor(H, S, D, P, g, seed=60 + S)
    w = orc.state_importance(cache, L, S, P, g, [0], nseg)
    Q, K = orc.widen_bf16(q)[0], orc.widen_bf16(k)[0]
    scale = orc.softmax_scale(D)
    parts = orc.partitions(S, P)
    tiles = orc.query_tiles(S, P)
    for t, (qpart, q0, q1) in enumerate(tiles):
        sets = orc.key_sets_of_tile(qpart, P, g)
        mass = np.zeros(nseg)
        for row in range(q0, q1):
            logits = [sum(Q[row][d] * K[j][d] for d in range(D)) * scale for j in range(S)]
            mx = max(logits)
            e = [math.exp(x - mx) for x in logits]
            tot = sum(e)
            for kk, ks in enumerate(sets):
                mass[kk] += sum(e[j] for p in ks for j in range(*parts[p])) / tot
        np.testing.assert_allclose(w[t], mass / (q1 - q0), rtol=1e-10, atol=1e-13)


@pytest.mark.parametrize("S,P,g", [(520, 4, 0), (700, 6, 2), (640, 8, 3)])
def test_importance_weights_sum_to_one(S, P, g):
    """Composition weights of all key sets of a row sum to one (Eq. 4)."""
    _, cache, L, nseg, _ = run_anchor(2, S, 8, P, g, seed=70 + S)
    w = orc.state_importance(cache, L, S, P, g, [0, 1], nseg)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=1e-12)
    assert np.all(w >= 0)


def second_statement(w_row, st_row, step, r, local):
    """Pick r times the smallest predicted error among the remaining
    candidates, the lower index on equal values."""
    left = [k for k in range(len(w_row)) if k != local and st_row[k] >= 0]
    row = [orc.COMPUTE] * len(w_row)
    for _ in range(min(r, len(left))):
        best = None
        for k in left:
            e = float(np.float32(w_row[k]) * np.float32(step - st_row[k]))
            if best is None or e < best[0]:
                best = (e, k)
        row[best[1]] = orc.REUSE
        left.remove(best[1])
    return row


def test_importance_rule_two_statements_agree():
    rng = np.random.default_rng(80)
    for trial in range(300):
        n = int(rng.integers(1, 17))
        w = rng.random(n).astype(np.float32)
        if trial % 3 == 0:                               # plenty of exact ties
            w = np.round(w * 4).astype(np.float32) / 4
        st = rng.integers(-1, 6, size=n)
        step = 7
        local = int(rng.integers(0, n))
        for r in range(n + 1):
            got = list(orc.importance_row(w, st, step, r, local))
            assert got == second_statement(w, st, step, r, local)
            assert got[local] == orc.COMPUTE
            assert all(got[k] == orc.COMPUTE for k in range(n) if st[k] < 0)


def test_importance_plan_prefers_small_weight_and_young_slots():
    # equal ages: the smallest weights are reused; equal weights: the
    # youngest slots (computed most recently) are reused first
    w = np.array([0.4, 0.1, 0.3, 0.2], dtype=np.float32)
    assert list(orc.importance_row(w, np.array([1, 1, 1, 1]), 3, 2, 0)) == [1, 0, 1, 0]
    w = np.full(4, 0.25, dtype=np.float32)
    assert list(orc.importance_row(w, np.array([1, 2, 1, 2]), 3, 2, 2)) == [1, 0, 1, 0]


def test_importance_plan_in_build_plan():
    H, S, D, P = 1, 512, 4, 4
    _, cache, L, nseg, st = run_anchor(H, S, D, P, 0, seed=81)
    w = orc.state_importance(cache, L, S, P, 0, [0], nseg).astype(np.float32)
    plan1, c1, _ = orc.build_plan(orc.MODE_IMPORTANCE, H, S, D, P, step=1, r=2, weights=w)
    assert np.all(plan1 == orc.COMPUTE) and c1["skipped_blocks"] == 0
    plan2, c2, st2 = orc.build_plan(orc.MODE_IMPORTANCE, H, S, D, P, step=2, r=2, weights=w, stamps=st)
    tiles = orc.query_tiles(S, P)
    for t, (qpart, _, _) in enumerate(tiles):
        assert plan2[t, qpart] == orc.COMPUTE and (plan2[t] == orc.REUSE).sum() == 2
        reused = [k for k in range(P) if plan2[t, k] == orc.REUSE]
        kept = [k for k in range(P) if plan2[t, k] == orc.COMPUTE and k != qpart]
        assert max(w[t, reused]) <= min(w[t, kept])
    assert c2["skipped_blocks"] == H * len(tiles) * 2 * 1
