"""Pins of the oracle's anchor-guided planner ("DiTango", selection strategy
and anchor steps): state errors, local drift, the anchor trigger, scale
ratios and the percentile threshold, each against a closed form or a second
independent statement."""

import math

import numpy as np
import pytest

import oracle as orc
from partitioned_attention_state_b200 import workloads as wl


def run_steps(H, S, D, P, sigmas, plans=None, seed=3):
    """Oracle steps with per-step perturbations sigmas[t] (steps 2, 3, ...):
    returns the list of (plan, diff, norm) and the final cache."""
    rng = np.random.Generator(np.random.PCG64(seed))
    master = [rng.standard_normal((H, S, D)).astype(np.float32) / np.float32(math.sqrt(D)) for _ in range(3)]
    cache = orc.StateCache()
    out = []
    nseg = P
    for t, sig in enumerate([0.0] + list(sigmas), start=1):
        if t > 1:
            for m in master:
                m += np.float32(sig) * rng.standard_normal(m.shape).astype(np.float32)
        q, k, v = (wl.f32_to_bf16_bits(m) for m in master)
        plan = plans[t - 1] if plans else np.full((len(orc.query_tiles(S, P)), nseg), orc.COMPUTE, np.uint8)
        before = dict(cache.slots)
        _, _, fresh = orc.partition_step(q, k, v, plan, S, P, cache)
        diff, norm = orc.state_errors(before, fresh, S, P, nseg)
        out.append((plan, diff, norm))
    return out, cache


def test_state_error_of_unchanged_inputs_is_zero_and_of_an_empty_cache_undefined():
    res, _ = run_steps(2, 512, 16, 4, [0.0, 0.0])
    _, d1, n1 = res[0]
    assert np.all(np.isnan(d1)) and np.all(np.isnan(n1))          # step 1: no previous state
    for _, d, n in res[1:]:
        assert np.all(d == 0.0) and np.all(n > 0.0)                  # identical inputs, identical states


def test_state_error_closed_forms():
    """e(fresh, cached) = ||fresh - cached|| / ||fresh||: a zero cached state
    gives exactly 1, a cached state equal to half the fresh one gives 1/2."""
    H, S, D, P = 1, 256, 8, 2
    res, cache = run_steps(H, S, D, P, [])
    before_zero = {key: (np.zeros_like(o), l) for key, (o, l) in cache.slots.items()}
    before_half = {key: (0.5 * o, l) for key, (o, l) in cache.slots.items()}
    fresh = {}
    for _, q0, q1 in orc.query_tiles(S, P):                      # one item per (key set, head, query tile)
        rs = np.arange(q0, q1)
        for (kk, h) in {(kk, h) for (kk, h, _) in cache.slots}:
            o, l = cache.get(kk, h, rs, D)
            fresh.setdefault((kk, h), []).append((rs, (o, l)))
    for before, want in ((before_zero, 1.0), (before_half, 0.5)):
        d, n = orc.state_errors(before, fresh, S, P, P)
        e = np.sqrt(d / n)
        np.testing.assert_allclose(e, want, rtol=1e-12)


def test_no_drift_no_anchor():
    """Zero perturbation: every local drift is exactly 0, so no anchor is
    triggered after step 1 however small theta is."""
    H, S, D, P = 2, 512, 16, 4
    nqt = len(orc.query_tiles(S, P))
    st = orc.AnchorState(nqt, P, rho=0.5, theta=1e-6)
    stamps = np.full((nqt, P), -1, np.int32)
    rng = np.random.Generator(np.random.PCG64(1))
    q, k, v = (wl.f32_to_bf16_bits(rng.standard_normal((H, S, D)).astype(np.float32) / 4) for _ in range(3))
    cache = orc.StateCache()
    for step in range(1, 6):
        plan, anchored = orc.anchor_plan(st, stamps, step, S, P)
        assert anchored == (step == 1)
        before_st = stamps.copy()
        before = dict(cache.slots)
        _, L, fresh = orc.partition_step(q, k, v, plan, S, P, cache)
        stamps[plan == orc.COMPUTE] = step
        d, n = orc.state_errors(before, fresh, S, P, P)
        w = orc.state_importance(cache, {(h, r): float(L[h, r]) for h in range(H) for r in range(S)}, S, P, 0,
                                 range(H), P) if anchored else None
        orc.anchor_update(st, step, anchored, before_st, d, n, S, P, w_now=w)
        assert np.all(st.drift == 0.0)


def test_large_perturbation_forces_an_anchor():
    """A perturbation far above the drift budget at step 3 makes step 4 an
    anchor; small ones before it do not."""
    H, S, D, P = 2, 512, 16, 4
    nqt = len(orc.query_tiles(S, P))
    st = orc.AnchorState(nqt, P, rho=0.5, theta=0.5)
    stamps = np.full((nqt, P), -1, np.int32)
    rng = np.random.Generator(np.random.PCG64(2))
    master = [rng.standard_normal((H, S, D)).astype(np.float32) / 4 for _ in range(3)]
    cache = orc.StateCache()
    anchors = []
    for step, sig in zip(range(1, 6), [0.0, 0.001, 2.0, 0.001, 0.001]):
        for m in master:
            m += np.float32(sig) * rng.standard_normal(m.shape).astype(np.float32)
        q, k, v = (wl.f32_to_bf16_bits(m) for m in master)
        plan, anchored = orc.anchor_plan(st, stamps, step, S, P)
        anchors.append(anchored)
        before_st = stamps.copy()
        before = dict(cache.slots)
        _, L, fresh = orc.partition_step(q, k, v, plan, S, P, cache)
        stamps[plan == orc.COMPUTE] = step
        d, n = orc.state_errors(before, fresh, S, P, P)
        w = orc.state_importance(cache, {(h, r): float(L[h, r]) for h in range(H) for r in range(S)}, S, P, 0,
                                 range(H), P) if anchored else None
        orc.anchor_update(st, step, anchored, before_st, d, n, S, P, w_now=w)
        if step == 3:
            assert np.all(st.drift > st.theta)
    assert anchors == [True, False, False, True, False]


@pytest.mark.parametrize("rho", [0.25, 0.5, 0.75, 1.0, 0.0])
def test_percentile_threshold_reuses_the_requested_count(rho):
    """Crafted errors with distinct rates w * alpha: at age 1 right after the
    anchor, exactly ceil(rho N) of the N (tile, non-local set) pairs are
    reused, and they are the ones of smallest rate."""
    S, P = 2048, 8
    nqt = len(orc.query_tiles(S, P))
    st = orc.AnchorState(nqt, P, rho=rho, theta=1.0)
    rng = np.random.Generator(np.random.PCG64(5))
    w = rng.uniform(0.01, 1.0, (nqt, P)).astype(np.float32)
    stamps_before = np.full((nqt, P), 1, np.int32)                # ages 1 at the anchor (step 2)
    e = rng.uniform(0.001, 0.1, (nqt, P))
    orc.anchor_update(st, 2, True, stamps_before, e ** 2, np.ones((nqt, P)), S, P, w_now=w)
    stamps = np.full((nqt, P), 2, np.int32)
    plan, anchored = orc.anchor_plan(st, stamps, 3, S, P)
    assert not anchored
    local = np.array([orc.query_tiles(S, P)[t][0] for t in range(nqt)])
    nonlocal_mask = np.ones((nqt, P), bool)
    nonlocal_mask[np.arange(nqt), local] = False
    n = int(nonlocal_mask.sum())
    assert int((plan == orc.REUSE).sum()) == math.ceil(rho * n)
    rate = w.astype(np.float64) * st.alpha
    if 0 < rho < 1:
        assert rate[(plan == orc.REUSE)].max() < rate[(plan == orc.COMPUTE) & nonlocal_mask].min()


def test_scale_ratio_is_error_per_step_of_age():
    S, P = 1024, 4
    nqt = len(orc.query_tiles(S, P))
    st = orc.AnchorState(nqt, P, rho=0.5, theta=1.0)
    stamps_before = np.array([[1, 3, -1, 2]] * nqt, np.int32)
    diff = np.full((nqt, P), 0.09)                                  # e = 0.3
    orc.anchor_update(st, 5, True, stamps_before, diff, np.ones((nqt, P)), S, P, w_now=np.ones((nqt, P)))
    for t in range(nqt):
        loc = orc.query_tiles(S, P)[t][0]
        for k, age in ((0, 4), (1, 2), (3, 3)):
            if k != loc:
                assert st.alpha[t, k] == np.float32(np.float32(0.3) / np.float32(age))
        assert st.alpha[t, 2] == 1.0 or 2 == loc                   # never cached: unmeasured


def test_selection_rule_second_statement():
    """The selection rule restated with vectorised numpy agrees with the
    oracle's loops on random metadata, including exact ties at epsilon."""
    S, P = 4096, 16
    tiles = orc.query_tiles(S, P)
    nqt = len(tiles)
    rng = np.random.Generator(np.random.PCG64(11))
    st = orc.AnchorState(nqt, P, rho=0.5, theta=10.0)
    st.w[:] = rng.choice([0.125, 0.25, 0.5], (nqt, P)).astype(np.float32)
    st.alpha[:] = rng.choice([0.5, 1.0, 2.0], (nqt, P)).astype(np.float32)
    st.eps = np.float32(0.5)
    stamps = rng.integers(-1, 6, (nqt, P)).astype(np.int32)
    step = 7
    plan, anchored = orc.anchor_plan(st, stamps, step, S, P)
    assert not anchored
    local = np.array([t[0] for t in tiles])
    ase = st.w * st.alpha * (step - stamps).astype(np.float32)
    want = np.where((ase <= st.eps) & (stamps >= 0), orc.REUSE, orc.COMPUTE).astype(np.uint8)
    want[np.arange(nqt), local] = orc.COMPUTE
    np.testing.assert_array_equal(plan, want)
