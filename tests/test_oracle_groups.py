"""Pins of the oracle's grouped state cache ("DiTango", state grouping and
Dynamic Group State Compose) against facts that do not come from the oracle:
the page's Fig. 6 example in grouped form, exact coverage of the keys, full
attention by brute force, agreement with the ungrouped path, and closed-form
block counts."""

import os

import numpy as np
import pytest

import oracle as orc
from partitioned_attention_state_b200 import workloads as wl

from test_oracle_pins import brute_state

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def read_grouped_golden():
    head, sets = {}, []
    with open(os.path.join(GOLDEN, "fig6_cp4_rank0_grouped.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            parts = line.split()
            if parts[0] == "set":
                sets.append(([int(x) for x in parts[2].split(",")], parts[3]))
            else:
                head[parts[0]] = int(parts[1])
    return head, sets


def test_fig6_grouped_golden():
    g, sets = read_grouped_golden()
    P, grp, q, r = g["P"], g["group"], g["query_partition"], g["reuse_groups"]
    assert orc.group_key_sets(q, P, grp) == [s for s, _ in sets]
    want = [orc.COMPUTE if d == "C" else orc.REUSE for _, d in sets]
    assert list(orc.group_proximity_row(q, P, grp, r)) == want
    # and from a full step-2 plan of the tiny geometry (query tiles of partition 0)
    plan, _, _ = orc.build_plan(orc.MODE_PROXIMITY, 2, 1024, 64, P, step=2, r=r, group=grp,
                                stamps=np.ones((8, 3), np.int32))
    assert plan.shape == (8, 3)
    assert list(plan[0]) == want and list(plan[1]) == want


@pytest.mark.parametrize("P", [1, 2, 3, 4, 5, 8, 16])
@pytest.mark.parametrize("g", [1, 2, 3, 4, 16])
def test_grouped_key_sets_cover_every_partition_once(P, g):
    m = -(-P // g)
    for q in range(P):
        sets = orc.group_key_sets(q, P, g)
        assert len(sets) == 1 + m and sets[0] == [q]
        flat = [k for s in sets for k in s]
        assert sorted(flat) == list(range(P))               # every partition exactly once
        for i, s in enumerate(sets[1:]):
            assert all(i * g <= k < (i + 1) * g for k in s)  # adjacent partitions of group i
            full = min((i + 1) * g, P) - i * g
            assert len(s) == full - (1 if i == q // g else 0)


def independent_group_row(q, P, g, r):
    """Second statement of the grouped proximity rule: walk group distances
    from the largest down, lower index first, reuse the first r groups."""
    m = -(-P // g)
    lg = q // g
    order = []
    for dist in range(m - 1, -1, -1):
        for i in sorted({lg - dist, lg + dist}):
            if 0 <= i < m:
                order.append(i)
    row = [orc.COMPUTE] * (1 + m)
    for i in order[:r]:
        row[1 + i] = orc.REUSE
    return row


@pytest.mark.parametrize("P,g", [(4, 2), (16, 4), (8, 3), (5, 2), (16, 1)])
def test_grouped_proximity_two_statements_agree(P, g):
    m = -(-P // g)
    for q in range(P):
        for r in range(m + 1):
            assert list(orc.group_proximity_row(q, P, g, r)) == independent_group_row(q, P, g, r)
            assert orc.group_proximity_row(q, P, g, r)[0] == orc.COMPUTE


@pytest.mark.parametrize("S,P,g", [(300, 3, 2), (520, 4, 2), (700, 5, 2), (640, 4, 4), (260, 2, 1)])
def test_grouped_anchor_step_is_full_attention(S, P, g):
    """Every key exactly once: the composed key sets of an all-compute step
    give softmax attention over the whole sequence (scalar loops)."""
    H, D = 1, 4
    q, k, v = wl.InputStream(H, S, D, sigma=0.05, seed=40 + S).next_step()
    plan, _, _ = orc.build_plan(orc.MODE_ALL_COMPUTE, H, S, D, P, step=1, group=g)
    rows = np.array([0, 1, S // 3, S // 2, S - 2, S - 1])
    o, l, _ = orc.partition_step(q, k, v, plan, S, P, orc.StateCache(), rows=rows, group=g)
    Q, K, V = orc.widen_bf16(q), orc.widen_bf16(k), orc.widen_bf16(v)
    fo, fl = brute_state(Q[0, rows], K[0], V[0], orc.softmax_scale(D))
    np.testing.assert_allclose(o[0], fo, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(l[0], fl, rtol=1e-12)


def test_grouped_reuse_with_unchanged_inputs_is_full_attention():
    """A reused composed state stands in for its group exactly: with the same
    inputs in both steps, every grouped plan reproduces the anchor output."""
    H, S, D, P, g = 2, 640, 8, 8, 2
    s = wl.InputStream(H, S, D, sigma=0.0, seed=41)
    q, k, v = s.next_step()
    cache = orc.StateCache()
    plan, _, st = orc.build_plan(orc.MODE_PROXIMITY, H, S, D, P, step=1, r=2, group=g)
    full, lfull, _ = orc.partition_step(q, k, v, plan, S, P, cache, group=g)
    for r in range(0, 5):
        plan2, c, _ = orc.build_plan(orc.MODE_PROXIMITY, H, S, D, P, step=2, r=r, group=g, stamps=st)
        assert (plan2 == orc.REUSE).sum() == r * len(plan2)
        o, l, _ = orc.partition_step(q, k, v, plan2, S, P, cache, group=g)
        np.testing.assert_allclose(o, full, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(l, lfull, rtol=1e-13)


def test_group_state_is_composition_of_partition_states():
    """Eq. 4 (associativity): the cached state of a group equals the
    composition of the per-partition states of its partitions."""
    H, S, D, P, g = 1, 768, 8, 6, 3
    q, k, v = wl.InputStream(H, S, D, sigma=0.05, seed=42).next_step()
    cp, cg = orc.StateCache(), orc.StateCache()
    pp, _, _ = orc.build_plan(orc.MODE_ALL_COMPUTE, H, S, D, P, step=1)
    pg, _, _ = orc.build_plan(orc.MODE_ALL_COMPUTE, H, S, D, P, step=1, group=g)
    orc.partition_step(q, k, v, pp, S, P, cp)
    orc.partition_step(q, k, v, pg, S, P, cg, group=g)
    for row in (0, 130, 300, 511, 767):
        qpart = row // 128
        for i, ks in enumerate(orc.group_key_sets(qpart, P, g)):
            got = cg.get(i, 0, [row], D)
            want = orc.compose_n([cp.get(kk, 0, [row], D) for kk in ks]) if ks else orc.identity_state(1, D)
            np.testing.assert_allclose(got[0], want[0], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(got[1], want[1], rtol=1e-13)


def test_group_size_one_equals_ungrouped_step():
    H, S, D, P, r = 1, 512, 4, 4, 2
    s = wl.InputStream(H, S, D, sigma=0.05, seed=43)
    c0, c1 = orc.StateCache(), orc.StateCache()
    st0 = st1 = None
    for step in (1, 2, 3):
        q, k, v = s.next_step()
        p0, n0, st0 = orc.build_plan(orc.MODE_PROXIMITY, H, S, D, P, step=step, r=r, stamps=st0)
        p1, n1, st1 = orc.build_plan(orc.MODE_PROXIMITY, H, S, D, P, step=step, r=r, group=1, stamps=st1)
        assert n0 == n1
        o0, l0, _ = orc.partition_step(q, k, v, p0, S, P, c0)
        o1, l1, _ = orc.partition_step(q, k, v, p1, S, P, c1, group=1)
        np.testing.assert_allclose(o1, o0, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(l1, l0, rtol=1e-13)


@pytest.mark.parametrize("g,r", [(4, 1), (4, 2), (4, 3), (2, 4), (8, 1)])
def test_grouped_counts_closed_form_video(g, r):
    """Video geometry (P = 16, all partitions 16 key tiles): a reuse step
    skips r groups of g partitions per query tile, unless the local group is
    among them (r = m), whose g - 1 partitions are then skipped."""
    w = wl.BY_NAME["video_21x30x52_h40_d128_p16"]
    m = 16 // g
    nqt = 256
    plan, c, _ = orc.build_plan(orc.MODE_PROXIMITY, w.H, w.S, w.D, w.P, step=2, r=r, group=g,
                                stamps=np.ones((nqt, 1 + m), np.int32))
    assert r < m
    assert c["skipped_blocks"] == w.H * nqt * r * g * 16
    assert c["computed_blocks"] == w.H * nqt * (16 - r * g) * 16
    _, c1, _ = orc.build_plan(orc.MODE_PROXIMITY, w.H, w.S, w.D, w.P, step=1, r=r, group=g)
    assert c1["computed_flops"] == 4 * w.H * w.D * w.S * w.S


def test_compose_groups_equals_direct_coarse_grouping():
    """Dynamic Group State Compose: composing the cached states of group size
    g pairwise gives the states that group size 2g computes directly, and a
    reuse step on the coarse layout reproduces full attention."""
    H, S, D, P, g = 1, 1024, 4, 8, 1
    s = wl.InputStream(H, S, D, sigma=0.0, seed=44)
    q, k, v = s.next_step()
    rows = np.arange(S)
    fine, coarse = orc.StateCache(), orc.StateCache()
    pf, _, stf = orc.build_plan(orc.MODE_ALL_COMPUTE, H, S, D, P, step=1, group=g)
    pc, _, _ = orc.build_plan(orc.MODE_ALL_COMPUTE, H, S, D, P, step=1, group=2 * g)
    full, lfull, _ = orc.partition_step(q, k, v, pf, S, P, fine, group=g)
    orc.partition_step(q, k, v, pc, S, P, coarse, group=2 * g)
    composed, st2 = orc.compose_groups(fine, stf, P, g, 2, [0], rows, S, D)
    assert st2.shape == (len(orc.query_tiles(S, P)), 1 + 4) and np.all(st2 == 1)
    for key, (o, l) in coarse.slots.items():
        o2, l2 = composed.slots[key]
        np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-14)
        assert abs(l2 - l) <= 1e-12 * max(1.0, abs(l)) or (l == l2)
    plan2, _, _ = orc.build_plan(orc.MODE_PROXIMITY, H, S, D, P, step=2, r=2, group=2 * g, stamps=st2)
    o, l, _ = orc.partition_step(q, k, v, plan2, S, P, composed, group=2 * g)
    np.testing.assert_allclose(o, full, rtol=1e-12, atol=1e-14)


def test_compose_groups_stamp_is_oldest():
    st = np.array([[5, 3, 4, -1, 2, 7]], dtype=np.int32)    # 1 tile, local + 5 groups
    _, st2 = orc.compose_groups(orc.StateCache(), st, 5, 1, 2, [], np.zeros(0, int), 128, 4)
    assert st2.tolist() == [[5, 3, -1, 7]]


# ------------------------------------------------------------ bf16 state cache

def test_bf16_cache_stores_representable_values_and_exact_lse():
    H, S, D, P = 1, 300, 8, 3
    q, k, v = wl.InputStream(H, S, D, sigma=0.05, seed=50).next_step()
    c32, c16 = orc.StateCache(), orc.StateCache(bf16=True)
    plan, _, _ = orc.build_plan(orc.MODE_ALL_COMPUTE, H, S, D, P, step=1)
    o32, l32, _ = orc.partition_step(q, k, v, plan, S, P, c32)
    o16, l16, _ = orc.partition_step(q, k, v, plan, S, P, c16)
    np.testing.assert_array_equal(o16, o32)            # the step's own output is not rounded
    for key, (o, l) in c16.slots.items():
        o_ref, l_ref = c32.slots[key]
        assert l == l_ref
        # every stored value is a bf16 value (8 significant bits) ...
        m, e = np.frexp(o)
        np.testing.assert_array_equal(np.ldexp(np.round(np.ldexp(m, 8)), e - 8), o)
        # ... within half a bf16 spacing of the exact one
        assert np.all(np.abs(o - o_ref) <= np.abs(o_ref) * 2.0 ** -8 + 1e-300)


def test_bf16_cache_reuse_error_within_rounding_bound():
    """With a bf16 cache and unchanged inputs, an all-REUSE step is a convex
    combination of states whose OUT elements each carry a rounding error of
    at most half a bf16 spacing, <= 2^-8 |x|, so it stays within 2^-8 max|OUT|
    of full attention."""
    H, S, D, P = 2, 640, 8, 5
    q, k, v = wl.InputStream(H, S, D, sigma=0.0, seed=51).next_step()
    cache = orc.StateCache(bf16=True)
    plan, _, st = orc.build_plan(orc.MODE_ALL_COMPUTE, H, S, D, P, step=1)
    full, lfull, _ = orc.partition_step(q, k, v, plan, S, P, cache)
    plan2, _, _ = orc.build_plan(orc.MODE_ALL_REUSE, H, S, D, P, step=2, stamps=st)
    o, l, _ = orc.partition_step(q, k, v, plan2, S, P, cache)
    np.testing.assert_allclose(l, lfull, rtol=1e-13)
    bound = 2.0 ** -8 * max(np.abs(st_o).max() for st_o, _ in cache.slots.values())
    assert np.abs(o - full).max() <= bound * (1 + 1e-9)
    assert np.abs(o - full).max() > 0                   # the rounding is really applied
