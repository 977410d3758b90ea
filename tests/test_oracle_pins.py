"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks the oracle against one of: a value printed on the pages
(tests/golden), a closed form, an invariant the pages state, a textbook or
library routine, or brute force written out with scalar Python loops.  Each
is chosen so that a plausible slip in the oracle (a dropped term, a sign, a
transposed operand, the wrong log base or scale) fails at least one of them.
"""

import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle as orc
from partitioned_attention_state_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand(shape, seed, scale=1.0):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape) * scale


# ---------------------------------------------------------------- brute force

def brute_state(q, k, v, scale, keep=None):
    """Scalar-loop softmax attention of every query row over a key set."""
    n, m, D = q.shape[0], k.shape[0], v.shape[1]
    out = np.zeros((n, D))
    lse = np.full(n, -math.inf)
    for i in range(n):
        logits = []
        for j in range(m):
            if keep is not None and not keep[i][j]:
                continue
            s = 0.0
            for d in range(q.shape[1]):
                s += q[i][d] * k[j][d]
            logits.append((s * scale, j))
        if not logits:
            continue
        mx = max(x for x, _ in logits)
        tot = sum(math.exp(x - mx) for x, _ in logits)
        for x, j in logits:
            w = math.exp(x - mx) / tot
            for d in range(D):
                out[i][d] += w * v[j][d]
        lse[i] = mx + math.log(tot)
    return out, lse


@pytest.mark.parametrize("n,m,D", [(3, 5, 4), (7, 2, 3), (1, 9, 6)])
def test_state_matches_brute_force(n, m, D):
    q, k, v = rand((n, D), 1), rand((m, D), 2), rand((m, D), 3)
    o, l = orc.attention_state(q, k, v, 0.7)
    bo, bl = brute_state(q, k, v, 0.7)
    np.testing.assert_allclose(o, bo, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l, bl, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("S,P", [(12, 1), (12, 2), (12, 3), (12, 4), (12, 6), (13, 4), (5, 4)])
def test_composed_partitions_equal_unpartitioned_brute_force(S, P):
    D = 3
    q, k, v = rand((S, D), 4), rand((S, D), 5), rand((S, D), 6)
    scale = orc.softmax_scale(D)
    states = [orc.attention_state(q, k[a:b], v[a:b], scale) for a, b in orc.partitions(S, P)]
    o, l = states[0]
    for st in states[1:]:
        o, l = orc.compose((o, l), st)
    bo, bl = brute_state(q, k, v, scale)
    np.testing.assert_allclose(o, bo, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l, bl, rtol=1e-12, atol=1e-13)
    on, ln = orc.compose_n(states)
    np.testing.assert_allclose(on, bo, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(ln, bl, rtol=1e-12, atol=1e-13)


def test_single_partition_equals_torch_sdpa_float64():
    """P = 1 reduces to plain softmax attention (library routine)."""
    S, D = 200, 72
    q, k, v = rand((S, D), 7), rand((S, D), 8), rand((S, D), 9)
    o, _ = orc.attention_state(q, k, v, orc.softmax_scale(D))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None],
        torch.from_numpy(v)[None, None])[0, 0].numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-12)
    lse_ref = torch.logsumexp(torch.from_numpy(q @ k.T) / math.sqrt(D), dim=1).numpy()
    np.testing.assert_allclose(orc.attention_state(q, k, v, 1 / math.sqrt(D))[1], lse_ref, rtol=1e-12)


# ------------------------------------------------------------- composition laws

def test_composition_associative_and_commutative():
    """[DT] states compose associatively and commutatively (Eq. 4)."""
    n, D, N = 6, 5, 5
    rng = np.random.Generator(np.random.PCG64(11))
    states = [(rng.standard_normal((n, D)), rng.standard_normal(n) * 4) for _ in range(N)]
    ref = orc.compose_n(states)
    for perm in list(itertools.permutations(range(N)))[::17]:
        # random bracketing: repeatedly merge a random adjacent pair
        items = [states[i] for i in perm]
        while len(items) > 1:
            j = int(rng.integers(len(items) - 1))
            items[j:j + 2] = [orc.compose(items[j], items[j + 1])]
        np.testing.assert_allclose(items[0][0], ref[0], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(items[0][1], ref[1], rtol=1e-13)


def test_identity_state_is_unit():
    n, D = 4, 3
    st = (rand((n, D), 12), rand(n, 13))
    e = orc.identity_state(n, D)
    for a, b in [(st, e), (e, st)]:
        o, l = orc.compose(a, b)
        np.testing.assert_array_equal(o, st[0])
        np.testing.assert_array_equal(l, st[1])
    o, l = orc.compose(e, e)
    assert np.all(o == 0) and np.all(l == -np.inf)


def test_compose_weights_by_exp_lse_two_keys():
    """Two single-key states: composing them is a 2-way softmax (closed form)."""
    a, b = 0.3, -1.1
    v1, v2 = np.array([[1.0, 0.0]]), np.array([[0.0, 1.0]])
    o, l = orc.compose((v1, np.array([a])), (v2, np.array([b])))
    w1 = math.exp(a) / (math.exp(a) + math.exp(b))
    np.testing.assert_allclose(o[0], [w1, 1 - w1], rtol=1e-14)
    np.testing.assert_allclose(l[0], math.log(math.exp(a) + math.exp(b)), rtol=1e-14)


# ----------------------------------------------------------------- closed forms

def test_zero_queries_give_log_n_and_mean():
    n, m, D = 3, 37, 8
    o, l = orc.attention_state(np.zeros((n, D)), rand((m, D), 14), v := rand((m, D), 15), 0.5)
    np.testing.assert_allclose(l, math.log(m), rtol=1e-15)
    np.testing.assert_allclose(o, np.tile(v.mean(axis=0), (n, 1)), rtol=1e-12, atol=1e-14)


def test_constant_values_pass_through():
    m, D = 20, 6
    row = rand(D, 16)
    o, _ = orc.attention_state(rand((4, D), 17), rand((m, D), 18), np.tile(row, (m, 1)), 1.0)
    np.testing.assert_allclose(o, np.tile(row, (4, 1)), rtol=1e-13)


def test_dominant_key_selects_its_value():
    D, m = 4, 10
    q = np.ones((1, D))
    k = np.zeros((m, D)); k[6] = 50.0 / D
    v = rand((m, D), 19)
    o, l = orc.attention_state(q, k, v, 1.0)
    np.testing.assert_allclose(o[0], v[6], rtol=1e-15, atol=1e-18)
    np.testing.assert_allclose(l[0], 50.0 + math.log(1 + 9 * math.exp(-50.0)), rtol=1e-15)


def test_empty_key_set_and_fully_masked_rows():
    o, l = orc.attention_state(rand((3, 4), 20), np.zeros((0, 4)), np.zeros((0, 4)), 1.0)
    assert np.all(o == 0) and np.all(l == -np.inf)
    keep = np.array([[True, False], [False, False]])
    o, l = orc.attention_state(rand((2, 4), 21), rand((2, 4), 22), v := rand((2, 4), 23), 1.0, keep)
    np.testing.assert_allclose(o[0], v[0], rtol=1e-15)
    assert np.all(o[1] == 0) and l[1] == -np.inf


def test_masked_state_matches_brute_force():
    S, D, W = 40, 3, 10
    q, k, v = rand((S, D), 24), rand((S, D), 25), rand((S, D), 26)
    inside = orc.window_in(np.arange(S), np.arange(S), W)
    assert inside[0, 5] and not inside[0, 6] and inside[20, 15] and not inside[20, 14]
    for keep in (inside, ~inside):
        o, l = orc.attention_state(q, k, v, 0.9, keep)
        bo, bl = brute_state(q, k, v, 0.9, keep)
        np.testing.assert_allclose(o, bo, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(l, bl, rtol=1e-12, atol=1e-13)


# -------------------------------------------------------------- plan and counts

def read_golden_plan():
    rows = {}
    with open(os.path.join(GOLDEN, "fig6_cp4_rank0.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            a, b = line.split()
            rows[a] = b
    return rows


def test_fig6_plan_row_golden():
    g = read_golden_plan()
    P, q, r = int(g["P"]), int(g["query_partition"]), int(g["reuse_per_row"])
    want = [orc.COMPUTE if g[str(k)] == "C" else orc.REUSE for k in range(P)]
    assert list(orc.proximity_row(q, P, r)) == want
    # the same row comes out of a full step-2 plan of the tiny workload
    plan, _, _ = orc.build_plan(orc.MODE_PROXIMITY, 2, 1024, 64, 4, step=2, r=2,
                                stamps=np.ones((8, 4), np.int32))
    assert list(plan[0]) == want and list(plan[1]) == want


def independent_proximity(P, r):
    """Second statement of the proximity rule: reuse the r largest distances,
    equal distances taken in index order; never the local partition."""
    out = []
    for q in range(P):
        order = []
        for dist in range(P - 1, 0, -1):
            for k in (q - dist, q + dist):
                if 0 <= k < P:
                    order.append(k)
        reuse = set(order[:r])
        out.append([orc.REUSE if k in reuse else orc.COMPUTE for k in range(P)])
    return np.array(out, dtype=np.uint8)


@pytest.mark.parametrize("P", [1, 2, 3, 4, 8, 16])
def test_proximity_rule_two_statements_agree(P):
    for r in range(P):
        ref = independent_proximity(P, r)
        got = np.stack([orc.proximity_row(q, P, r) for q in range(P)])
        np.testing.assert_array_equal(got, ref)
        assert np.all(np.diag(got) == orc.COMPUTE)
        assert np.all((got == orc.REUSE).sum(axis=1) == r)


def test_tiny_plan_rows():
    got = np.stack([orc.proximity_row(q, 4, 2) for q in range(4)])
    np.testing.assert_array_equal(got, [[1, 1, 0, 0], [0, 1, 1, 0], [0, 0, 1, 1], [0, 0, 1, 1]])


def test_partition_geometry_video():
    parts = orc.partitions(32760, 16)
    assert [b - a for a, b in parts] == [2048] * 15 + [2040]
    tiles = orc.query_tiles(32760, 16)
    assert len(tiles) == 256 and tiles[-1] == (15, 32640, 32760)
    assert orc.partitions(5, 4) == [(0, 2), (2, 4), (4, 5), (5, 5)]


EXPECTED_COUNTS = {
    # (workload, r): (computed_blocks, skipped_blocks) of a reuse step, from
    # H * nqt * (P - r) * kv_tiles_per_partition (all partitions equal-tiled)
    (0, 2): (2 * 8 * 2 * 2, 2 * 8 * 2 * 2),
    (1, 0): (16 * 8 * 8 * 1, 0), (1, 2): (16 * 8 * 6, 16 * 8 * 2),
    (1, 4): (16 * 8 * 4, 16 * 8 * 4), (1, 6): (16 * 8 * 2, 16 * 8 * 6),
    (2, 8): (16 * 128 * 8 * 8, 16 * 128 * 8 * 8),
    (3, 0): (40 * 256 * 16 * 16, 0), (3, 4): (40 * 256 * 12 * 16, 40 * 256 * 4 * 16),
    (3, 8): (40 * 256 * 8 * 16, 40 * 256 * 8 * 16), (3, 12): (40 * 256 * 4 * 16, 40 * 256 * 12 * 16),
}


@pytest.mark.parametrize("key", sorted(EXPECTED_COUNTS))
def test_counts_closed_form(key):
    wi, r = key
    w = wl.WORKLOADS[wi]
    nqt = len(orc.query_tiles(w.S, w.P))
    plan, c, st = orc.build_plan(orc.MODE_PROXIMITY, w.H, w.S, w.D, w.P, step=2, r=r,
                                 stamps=np.ones((nqt, w.P), np.int32))
    assert (c["computed_blocks"], c["skipped_blocks"]) == EXPECTED_COUNTS[key]
    assert np.all(st[plan == orc.COMPUTE] == 2) and np.all(st[plan == orc.REUSE] == 1)
    # algorithmic FLOPs: every computed pair of a (tile, partition) block
    parts = orc.partitions(w.S, w.P)
    tiles = orc.query_tiles(w.S, w.P)
    fl = sum(4 * w.H * w.D * (q1 - q0) * (parts[k][1] - parts[k][0])
             for t, (_, q0, q1) in enumerate(tiles) for k in range(w.P) if plan[t, k])
    assert c["computed_flops"] == fl
    # anchor step computes everything: full attention flops 4 H D S^2
    _, c1, _ = orc.build_plan(orc.MODE_PROXIMITY, w.H, w.S, w.D, w.P, step=1, r=r)
    assert c1["computed_flops"] == 4 * w.H * w.D * w.S * w.S and c1["skipped_blocks"] == 0


def test_window_counts_closed_form():
    w = wl.WORKLOADS[4]
    hw = w.window // 2
    _, c, _ = orc.build_plan(orc.MODE_WINDOW, w.H, w.S, w.D, 1, step=2, window=w.window,
                             stamps=np.ones((128, 2), np.int32))
    # band blocks of query tile i: key tiles i-4..i+4 clipped to [0, 128)
    band = sum(min(127, i + 4) - max(0, i - 4) + 1 for i in range(128))
    assert band == 1132
    assert c["computed_blocks"] == w.H * band
    assert c["skipped_blocks"] == w.H * (128 * 128 - band)
    # in-window pairs: 1025 keys per interior row, clipped at both ends
    pairs = sum(min(w.S - 1, i + hw) - max(0, i - hw) + 1 for i in range(w.S))
    assert pairs == 1025 * w.S - 2 * sum(range(1, hw + 1))
    assert c["computed_flops"] == 4 * w.H * w.D * pairs
    _, c1, _ = orc.build_plan(orc.MODE_WINDOW, w.H, w.S, w.D, 1, step=1, window=w.window)
    assert c1["computed_blocks"] == w.H * 128 * 128 and c1["skipped_blocks"] == 0


def test_reuse_of_empty_slot_is_refused():
    with pytest.raises(orc.CacheEmpty):
        orc.build_plan(orc.MODE_ALL_REUSE, 2, 1024, 64, 4, step=2)
    with pytest.raises(orc.CacheEmpty):
        orc.build_plan(orc.MODE_PROXIMITY, 2, 1024, 64, 4, step=2, r=1)


# ------------------------------------------------------ step-level invariants

def small_inputs(H, S, D, seed):
    return wl.InputStream(H, S, D, sigma=0.05, seed=seed)


def test_all_reuse_with_same_inputs_reproduces_full_attention():
    """[DT] a reused state replaces the exact remote computation."""
    H, S, D, P = 2, 300, 8, 3
    q, k, v = small_inputs(H, S, D, 30).next_step()
    cache = orc.StateCache()
    plan1, _, st = orc.build_plan(orc.MODE_ALL_COMPUTE, H, S, D, P, step=1)
    o1, l1, _ = orc.partition_step(q, k, v, plan1, S, P, cache)
    plan2, _, _ = orc.build_plan(orc.MODE_ALL_REUSE, H, S, D, P, step=2, stamps=st)
    o2, l2, fresh = orc.partition_step(q, k, v, plan2, S, P, cache)
    assert fresh == {}
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-14)
    Q, K, V = orc.widen_bf16(q), orc.widen_bf16(k), orc.widen_bf16(v)
    for h in range(H):
        fo, fl = brute_state(Q[h, ::37], K[h], V[h], orc.softmax_scale(D))
        np.testing.assert_allclose(o2[h, ::37], fo, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(l2[h, ::37], fl, rtol=1e-12)


def test_zero_perturbation_any_plan_is_exact():
    H, S, D, P = 1, 256, 4, 4
    s = wl.InputStream(H, S, D, sigma=0.0, seed=31)
    q, k, v = s.next_step()
    cache = orc.StateCache()
    plan, _, st = orc.build_plan(orc.MODE_PROXIMITY, H, S, D, P, step=1, r=2)
    full, _, _ = orc.partition_step(q, k, v, plan, S, P, cache)
    q2, k2, v2 = s.next_step()
    assert np.array_equal(q2, q)
    for r in range(P):
        plan, _, _ = orc.build_plan(orc.MODE_PROXIMITY, H, S, D, P, step=2, r=r, stamps=st)
        o, _, _ = orc.partition_step(q2, k2, v2, plan, S, P, cache)
        np.testing.assert_allclose(o, full, rtol=1e-12, atol=1e-14)


def test_sampled_rows_agree_with_full_run():
    H, S, D, P = 2, 520, 8, 4
    s = small_inputs(H, S, D, 32)
    rows = np.array([0, 5, 127, 128, 129, 260, 519])
    c_full, c_rows = orc.StateCache(), orc.StateCache()
    st = None
    for step in (1, 2):
        q, k, v = s.next_step()
        plan, _, st = orc.build_plan(orc.MODE_PROXIMITY, H, S, D, P, step=step, r=2, stamps=st)
        of, lf, _ = orc.partition_step(q, k, v, plan, S, P, c_full)
        orow, lrow, _ = orc.partition_step(q, k, v, plan, S, P, c_rows, rows=rows)
        # same arithmetic; only the BLAS blocking of the row subset differs
        np.testing.assert_allclose(orow, of[:, rows], rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(lrow, lf[:, rows], rtol=1e-14)


def test_window_plus_residual_same_step_is_full_attention():
    """[DFA] window + (full - window) at the same step is full attention."""
    H, S, D, W = 1, 300, 8, 64
    q, k, v = small_inputs(H, S, D, 33).next_step()
    R = {}
    o1, l1 = orc.window_step(q, k, v, W, True, R)
    o2, _ = orc.window_step(q, k, v, W, False, R)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-13)
    Q, K, V = orc.widen_bf16(q), orc.widen_bf16(k), orc.widen_bf16(v)
    fo, fl = brute_state(Q[0, ::29], K[0], V[0], orc.softmax_scale(D))
    np.testing.assert_allclose(o1[0, ::29], fo, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(l1[0, ::29], fl, rtol=1e-12)
    # window attention itself against brute force with the band mask
    rows = np.arange(0, S, 29)
    keep = orc.window_in(rows, np.arange(S), W)
    wo, wlse = orc.attention_state(Q[0, rows], K[0], V[0], orc.softmax_scale(D), keep)
    bo, bl = brute_state(Q[0, rows], K[0], V[0], orc.softmax_scale(D), keep)
    np.testing.assert_allclose(wo, bo, rtol=1e-11, atol=1e-12)
    o3, l3 = orc.window_step(q, k, v, W, False, R, rows=rows)
    np.testing.assert_allclose(l3[0], bl, rtol=1e-12)


def test_wide_window_is_full_attention_and_zero_residual():
    H, S, D = 1, 200, 4
    q, k, v = small_inputs(H, S, D, 34).next_step()
    R = {}
    o1, _ = orc.window_step(q, k, v, 2 * S, True, R)
    assert max(np.abs(r).max() for r in R.values()) < 1e-15
    plan, _, _ = orc.build_plan(orc.MODE_ALL_COMPUTE, H, S, D, 1, step=1)
    o2, _, _ = orc.partition_step(q, k, v, plan, S, 1, orc.StateCache())
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-15)


# ------------------------------------------------------------------ bf16 bytes

def test_bf16_round_and_widen_match_torch():
    x = np.random.Generator(np.random.PCG64(40)).standard_normal(10000).astype(np.float32)
    x[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 0.0]   # ties
    bits = wl.f32_to_bf16_bits(x)
    tb = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bits, tb)
    np.testing.assert_array_equal(orc.widen_bf16(bits),
                                  torch.from_numpy(tb.view(np.int16)).view(torch.bfloat16).double().numpy())
    np.testing.assert_array_equal(orc.round_bf16(x.astype(np.float64)), orc.widen_bf16(bits))
