"""C-ABI library checks that need no GPU: exports, host plan builder against
the oracle (bit-exact), status codes and argument validation."""

import os
import re

import numpy as np
import pytest

import oracle as orc
import partitioned_attention_state_b200 as dt
from partitioned_attention_state_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"^DT_API\s+[\w\s\*]+?\b(dt_\w+)\s*\(", text, re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    lib = dt.load()
    names = header_functions()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    for s in (dt.DT_OK, dt.DT_ERR_INVALID, dt.DT_ERR_UNSUPPORTED, dt.DT_ERR_CACHE_EMPTY, dt.DT_ERR_CUDA,
              dt.DT_ERR_TIMEOUT):
        assert dt.dt_status_string(s).startswith("DT_")
    assert "unknown" in dt.dt_status_string(12345)


def run_both(mode, H, S, D, P, step, r=0, window=0, stamps=None, explicit=None, group=0):
    p = dt.params(H, S, D, P, mode, r, window, step, group)
    st_c = None if stamps is None else stamps.copy()
    plan_c, counts_c = dt.dt_plan_build(p, st_c, explicit)
    plan_o, counts_o, st_o = orc.build_plan(mode, H, S, D, P if mode != orc.MODE_WINDOW else 1, step, r=r,
                                            window=window, stamps=stamps, explicit=explicit, group=group)
    np.testing.assert_array_equal(plan_c, plan_o)
    assert counts_c == counts_o
    if st_c is not None:
        np.testing.assert_array_equal(st_c, st_o)
    return plan_c, counts_c, st_c


@pytest.mark.parametrize("wi", range(len(wl.WORKLOADS)))
def test_plan_matches_oracle_on_every_workload_schedule(wi):
    w = wl.WORKLOADS[wi]
    mode = orc.MODE_WINDOW if w.window else orc.MODE_PROXIMITY
    for r in w.reuse:
        p = dt.params(w.H, w.S, w.D, w.P, mode, r, w.window, 1)
        nqt, nseg = dt.dt_plan_geometry(p)
        stamps = np.full((nqt, nseg), -1, np.int32)
        for step in range(1, w.steps + 1):
            _, _, stamps = run_both(mode, w.H, w.S, w.D, w.P, step, r=r, window=w.window, stamps=stamps)


@pytest.mark.parametrize("S,P,r", [(1000, 3, 1), (5, 4, 2), (130, 1, 0), (257, 2, 1), (4097, 7, 5), (300, 5, 4)])
def test_plan_matches_oracle_ragged_geometry(S, P, r):
    H, D = 3, 64
    p = dt.params(H, S, D, P, dt.DT_MODE_PROXIMITY, r, 0, 1)
    nqt, nseg = dt.dt_plan_geometry(p)
    assert nqt == len(orc.query_tiles(S, P))
    st = np.full((nqt, nseg), -1, np.int32)
    _, _, st = run_both(orc.MODE_PROXIMITY, H, S, D, P, 1, r=r, stamps=st)
    run_both(orc.MODE_PROXIMITY, H, S, D, P, 2, r=r, stamps=st)
    run_both(orc.MODE_ALL_REUSE, H, S, D, P, 3, stamps=st)
    ex = (np.arange(nqt * nseg).reshape(nqt, nseg) % 3 == 0).astype(np.uint8)
    run_both(orc.MODE_EXPLICIT, H, S, D, P, 3, stamps=st, explicit=ex)


@pytest.mark.parametrize("S,W", [(16384, 1024), (1000, 100), (300, 64), (129, 1), (200, 400), (5000, 129)])
def test_window_plan_matches_oracle(S, W):
    st = None
    for step in (1, 2, 3):
        p = dt.params(2, S, 72, 1, dt.DT_MODE_WINDOW, 0, W, step)
        nqt, nseg = dt.dt_plan_geometry(p)
        assert nseg == 2
        if st is None:
            st = np.full((nqt, nseg), -1, np.int32)
        _, _, st = run_both(orc.MODE_WINDOW, 2, S, 72, 1, step, window=W, stamps=st)


def test_fig6_row_through_c_abi():
    p = dt.params(2, 1024, 64, 4, dt.DT_MODE_PROXIMITY, 2, 0, 2)
    plan, counts = dt.dt_plan_build(p, np.ones((8, 4), np.int32))
    assert list(plan[0]) == [1, 1, 0, 0]
    assert (counts["computed_blocks"], counts["skipped_blocks"]) == (64, 64)


def test_reuse_without_cache_is_refused_and_stamps_untouched():
    p = dt.params(2, 1024, 64, 4, dt.DT_MODE_PROXIMITY, 2, 0, 2)
    st = np.full((8, 4), -1, np.int32)
    with pytest.raises(dt.DtError) as e:
        dt.dt_plan_build(p, st)
    assert e.value.status == dt.DT_ERR_CACHE_EMPTY
    assert np.all(st == -1)
    with pytest.raises(dt.DtError):
        dt.dt_plan_build(dt.params(2, 1024, 64, 4, dt.DT_MODE_ALL_REUSE, 0, 0, 1), None)


@pytest.mark.parametrize("bad", [
    dict(P=0), dict(S=-1), dict(step=0), dict(mode=7), dict(r=4), dict(r=-1), dict(mode=4, window=0),
])
def test_invalid_plan_params(bad):
    kw = dict(H=2, S=1024, D=64, P=4, mode=dt.DT_MODE_PROXIMITY, r=1, window=0, step=1)
    kw.update(bad)
    p = dt.params(kw["H"], kw["S"], kw["D"], kw["P"], kw["mode"], kw["r"], kw["window"], kw["step"])
    with pytest.raises(dt.DtError) as e:
        dt.dt_plan_build(p)
    assert e.value.status == dt.DT_ERR_INVALID


def test_explicit_plan_value_checked():
    p = dt.params(1, 256, 64, 2, dt.DT_MODE_EXPLICIT, 0, 0, 1)
    with pytest.raises(dt.DtError):
        dt.dt_plan_build(p, None, np.full((2, 2), 7, np.uint8))


def test_empty_sequence_has_no_tiles():
    p = dt.params(4, 0, 64, 4, dt.DT_MODE_PROXIMITY, 1, 0, 1)
    assert dt.dt_plan_geometry(p)[0] == 0
    plan, counts = dt.dt_plan_build(p)
    assert plan.size == 0 and counts == {"computed_blocks": 0, "skipped_blocks": 0, "computed_flops": 0}


def test_device_entry_points_validate_before_any_cuda_call():
    """These argument errors are caught on the host, so they run without a GPU."""
    p = dt.params(2, 1024, 96, 4, dt.DT_MODE_PROXIMITY, 1, 0, 1)
    lib = dt.load()
    import ctypes
    assert lib.dt_attn_partial_fused(ctypes.byref(p), *([None] * 11), None) == dt.DT_ERR_UNSUPPORTED
    p.D = 64
    assert lib.dt_attn_partial_fused(ctypes.byref(p), *([None] * 11), None) == dt.DT_ERR_INVALID
    p.H = 0
    assert lib.dt_attn_partial_fused(ctypes.byref(p), *([None] * 11), None) == dt.DT_OK
    assert lib.dt_state_merge(0, 1, 1, 64, None, None, None, None, None, None) == dt.DT_ERR_INVALID
    assert lib.dt_state_merge(2, 1, 1, 66, None, None, None, None, None, None) == dt.DT_ERR_INVALID
    assert lib.dt_window_residual(5, 1, 1, 64, None, None, None, None, None, None) == dt.DT_ERR_INVALID
    assert lib.dt_window_residual(0, 1, 8, 64, None, None, None, None, None, None) == dt.DT_ERR_INVALID
    pw = dt.params(1, 64, 64, 1, dt.DT_MODE_WINDOW, 0, 8, 1)
    assert lib.dt_state_cache_update(ctypes.byref(pw), *([None] * 7)) == dt.DT_ERR_INVALID
    # the fused kernel keeps a plan row as a 64-bit mask: at most 64 partitions
    p64 = dt.params(1, 128 * 65, 64, 65, dt.DT_MODE_ALL_COMPUTE, 0, 0, 1)
    assert lib.dt_attn_partial_fused(ctypes.byref(p64), *([None] * 11), None) == dt.DT_ERR_UNSUPPORTED
    p64.P = 64
    assert lib.dt_attn_partial_fused(ctypes.byref(p64), *([None] * 11), None) == dt.DT_ERR_INVALID  # null buffers
    # misaligned device pointers (the plan included) are refused on the host
    p = dt.params(1, 128, 64, 1, dt.DT_MODE_ALL_COMPUTE, 0, 0, 1)
    plan_fake = [16 * 1024 + 4] + [16 * 1024] * 9
    assert lib.dt_attn_partial_fused(ctypes.byref(p), *plan_fake, 16 * 1024, None) == dt.DT_ERR_UNSUPPORTED
    fake = [16 * 1024] * 10
    fake[1] = 16 * 1024 + 2
    assert lib.dt_attn_partial_fused(ctypes.byref(p), *fake, 16 * 1024, None) == dt.DT_ERR_UNSUPPORTED


def test_head_range_validated_on_the_host():
    """dt_attn_partial_fused_heads refuses ranges outside [0, H) before any
    CUDA call; an empty range launches nothing."""
    import ctypes
    lib = dt.load()
    p = dt.params(3, 1024, 64, 4, dt.DT_MODE_PROXIMITY, 1, 0, 1)
    for h0, n in ((-1, 1), (0, -1), (1, 3), (3, 1), (0, 4)):
        assert lib.dt_attn_partial_fused_heads(ctypes.byref(p), h0, n, *([None] * 11), None) == dt.DT_ERR_INVALID
    for h0 in (0, 2, 3):
        assert lib.dt_attn_partial_fused_heads(ctypes.byref(p), h0, 0, *([None] * 11), None) == dt.DT_OK
    # a valid range still needs its buffers
    assert lib.dt_attn_partial_fused_heads(ctypes.byref(p), 1, 2, *([None] * 11), None) == dt.DT_ERR_INVALID
    assert lib.dt_attn_partial_fused_heads(None, 0, 1, *([None] * 11), None) == dt.DT_ERR_INVALID


@pytest.mark.parametrize("S,P,g,r", [(32760, 16, 4, 2), (16384, 16, 4, 1), (1024, 8, 2, 2), (1000, 3, 2, 1),
                                     (5, 4, 3, 1), (4097, 7, 3, 2), (300, 5, 1, 4), (2600, 64, 8, 3),
                                     (640, 4, 4, 1), (130, 2, 2, 1)])
def test_grouped_plan_matches_oracle(S, P, g, r):
    """State grouping: geometry, plans, counts and stamps of the C builder
    equal the oracle's, bit for bit, through a schedule of every mode."""
    H, D = 3, 64
    p = dt.params(H, S, D, P, dt.DT_MODE_PROXIMITY, r, 0, 1, g)
    nqt, nseg = dt.dt_plan_geometry(p)
    assert nqt == len(orc.query_tiles(S, P)) and nseg == 1 + -(-P // g)
    st = np.full((nqt, nseg), -1, np.int32)
    _, _, st = run_both(orc.MODE_PROXIMITY, H, S, D, P, 1, r=r, stamps=st, group=g)
    _, c2, st = run_both(orc.MODE_PROXIMITY, H, S, D, P, 2, r=r, stamps=st, group=g)
    run_both(orc.MODE_ALL_REUSE, H, S, D, P, 3, stamps=st, group=g)
    ex = (np.arange(nqt * nseg).reshape(nqt, nseg) % 3 == 0).astype(np.uint8)
    run_both(orc.MODE_EXPLICIT, H, S, D, P, 3, stamps=st, explicit=ex, group=g)
    _, call, _ = run_both(orc.MODE_ALL_COMPUTE, H, S, D, P, 4, group=g)
    # grouping only regroups the blocks: the anchor computes every block once
    _, cflat = dt.dt_plan_build(dt.params(H, S, D, P, dt.DT_MODE_ALL_COMPUTE, 0, 0, 1), None)
    assert call == cflat


def test_grouped_params_validated():
    import ctypes
    lib = dt.load()
    nqt, nseg = ctypes.c_int32(), ctypes.c_int32()
    bad = [dt.params(1, 1024, 64, 16, dt.DT_MODE_PROXIMITY, 5, 0, 1, 4),   # r > m = 4
           dt.params(1, 1024, 64, 16, dt.DT_MODE_PROXIMITY, 1, 0, 1, -1),
           dt.params(1, 1024, 64, 1, dt.DT_MODE_WINDOW, 0, 64, 1, 2)]      # grouping is for partitions
    for p in bad:
        assert lib.dt_plan_geometry(ctypes.byref(p), ctypes.byref(nqt), ctypes.byref(nseg)) == dt.DT_ERR_INVALID
    ok = dt.params(1, 1024, 64, 16, dt.DT_MODE_PROXIMITY, 4, 0, 1, 4)        # r = m: the local group too
    assert lib.dt_plan_geometry(ctypes.byref(ok), ctypes.byref(nqt), ctypes.byref(nseg)) == dt.DT_OK
    # the fused kernel keeps a plan row as a 64-bit mask: at most 64 key sets
    p = dt.params(1, 128 * 130, 64, 130, dt.DT_MODE_ALL_COMPUTE, 0, 0, 1, 2)   # 1 + 65 sets
    assert lib.dt_attn_partial_fused(ctypes.byref(p), *([None] * 11), None) == dt.DT_ERR_UNSUPPORTED
    p.group = 3                                                             # 1 + 44 sets
    assert lib.dt_attn_partial_fused(ctypes.byref(p), *([None] * 11), None) == dt.DT_ERR_INVALID


@pytest.mark.parametrize("P,g,f", [(16, 1, 2), (16, 2, 2), (16, 4, 2), (8, 1, 3), (5, 1, 2), (7, 2, 4), (16, 1, 8)])
def test_group_compose_stamps_match_oracle(P, g, f):
    """Host half of Dynamic Group State Compose (H = 0: no device work): the
    stamps of the coarse layout equal the oracle's, and the coarse layout's
    geometry is that of group size g * f."""
    S = 128 * P
    p = dt.params(0, S, 64, P, dt.DT_MODE_PROXIMITY, 0, 0, 1, g)
    nqt, nseg = dt.dt_plan_geometry(p)
    rng = np.random.default_rng(P * 100 + g * 10 + f)
    st = rng.integers(-1, 9, size=(nqt, nseg)).astype(np.int32)
    _, want = orc.compose_groups(orc.StateCache(), st, P, g, f, [], np.zeros(0, int), S, 64)
    got = dt.dt_group_compose(p, f, st.copy(), None, None, stream=0)
    np.testing.assert_array_equal(got, want)
    assert got.shape[1] == dt.dt_plan_geometry(dt.params(0, S, 64, P, dt.DT_MODE_PROXIMITY, 0, 0, 1, g * f))[1]


def test_group_compose_validated():
    import ctypes
    lib = dt.load()
    p = dt.params(2, 1024, 64, 8, dt.DT_MODE_PROXIMITY, 0, 0, 1, 2)
    assert lib.dt_group_compose(ctypes.byref(p), 1, None, None, None, None, None) == dt.DT_ERR_INVALID  # factor
    assert lib.dt_group_compose(ctypes.byref(p), 2, None, None, None, None, None) == dt.DT_ERR_INVALID  # no cache
    p.group = 0
    assert lib.dt_group_compose(ctypes.byref(p), 2, None, None, None, None, None) == dt.DT_ERR_INVALID  # ungrouped
    p.group, p.D = 2, 66
    assert lib.dt_group_compose(ctypes.byref(p), 2, None, None, None, None, None) == dt.DT_ERR_INVALID
    p.D = 64
    assert lib.dt_group_compose(ctypes.byref(p), 2, None, 16 * 1024 + 4, 16 * 1024, None, None) == \
        dt.DT_ERR_UNSUPPORTED



def test_state_dtype_validated():
    import ctypes
    lib = dt.load()
    p = dt.params(1, 1024, 64, 4, dt.DT_MODE_PROXIMITY, 1, 0, 1, 0, 2)          # unknown state type
    assert lib.dt_attn_partial_fused(ctypes.byref(p), *([None] * 11), None) == dt.DT_ERR_INVALID
    pw = dt.params(1, 1024, 64, 1, dt.DT_MODE_WINDOW, 0, 64, 1, 0, dt.DT_STATE_BF16)   # no cache in window mode
    assert lib.dt_attn_partial_fused(ctypes.byref(pw), *([None] * 11), None) == dt.DT_ERR_INVALID
    pb = dt.params(1, 1024, 64, 4, dt.DT_MODE_PROXIMITY, 1, 0, 1, 0, dt.DT_STATE_BF16)
    assert lib.dt_attn_partial_fused(ctypes.byref(pb), *([None] * 11), None) == dt.DT_ERR_INVALID  # null buffers
    assert lib.dt_state_cache_update(ctypes.byref(pb), *([None] * 7)) == dt.DT_ERR_UNSUPPORTED
    pb.group = 2
    assert lib.dt_group_compose(ctypes.byref(pb), 2, None, None, None, None, None) == dt.DT_ERR_UNSUPPORTED
    # the plan does not depend on the state type
    a, ca = dt.dt_plan_build(dt.params(1, 1024, 64, 4, dt.DT_MODE_PROXIMITY, 1, 0, 1), None)
    b, cb = dt.dt_plan_build(dt.params(1, 1024, 64, 4, dt.DT_MODE_PROXIMITY, 1, 0, 1, 0, dt.DT_STATE_BF16), None)
    assert np.array_equal(a, b) and ca == cb


@pytest.mark.parametrize("S,P,g", [(1024, 4, 0), (2600, 7, 0), (32760, 16, 4), (1800, 12, 5), (640, 8, 1)])
def test_importance_plan_matches_oracle(S, P, g):
    """dt_plan_build_importance against the oracle's rule, bit for bit, on
    random weights with exact ties and random stamps (never-written slots
    included), through steps 1-3."""
    H, D = 2, 64
    p = dt.params(H, S, D, P, dt.DT_MODE_IMPORTANCE, 2, 0, 1, g)
    nqt, nseg = dt.dt_plan_geometry(p)
    rng = np.random.default_rng(S + P + g)
    w = rng.random((nqt, nseg)).astype(np.float32)
    w[::3] = np.round(w[::3] * 4) / 4                       # exact ties
    for r in (0, 1, 2, nseg - 1):
        st = rng.integers(-1, 3, size=(nqt, nseg)).astype(np.int32)
        st_o = st.copy()
        for step in (1, 2, 3):
            p = dt.params(H, S, D, P, dt.DT_MODE_IMPORTANCE, r, 0, step, g)
            plan_c, counts_c = dt.dt_plan_build_importance(p, w, st)
            plan_o, counts_o, st_o = orc.build_plan(orc.MODE_IMPORTANCE, H, S, D, P, step, r=r, stamps=st_o,
                                                    group=g, weights=w)
            np.testing.assert_array_equal(plan_c, plan_o)
            assert counts_c == counts_o
            np.testing.assert_array_equal(st, st_o)


def test_importance_calls_validated():
    import ctypes
    lib = dt.load()
    p = dt.params(1, 1024, 64, 4, dt.DT_MODE_IMPORTANCE, 1, 0, 2)
    nqt, nseg = dt.dt_plan_geometry(p)
    plan = np.zeros((nqt, nseg), np.uint8)
    out = dt.Plan()
    out.plan = plan.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))
    assert lib.dt_plan_build(ctypes.byref(p), None, ctypes.byref(out)) == dt.DT_ERR_INVALID       # needs weights
    assert lib.dt_plan_build_importance(ctypes.byref(p), None, ctypes.byref(out)) == dt.DT_ERR_INVALID
    p.step = 1                                                                                        # anchor: no weights needed
    assert lib.dt_plan_build_importance(ctypes.byref(p), None, ctypes.byref(out)) == dt.DT_OK and plan.all()
    pp = dt.params(1, 1024, 64, 4, dt.DT_MODE_PROXIMITY, 1, 0, 2)
    w = np.ones((nqt, nseg), np.float32)
    assert lib.dt_plan_build_importance(ctypes.byref(pp), w.ctypes.data, ctypes.byref(out)) == dt.DT_ERR_INVALID
    p.reuse_per_row, p.step = 4, 2                                                                    # r > P - 1
    assert lib.dt_plan_build_importance(ctypes.byref(p), w.ctypes.data, ctypes.byref(out)) == dt.DT_ERR_INVALID
    pw = dt.params(1, 1024, 64, 1, dt.DT_MODE_WINDOW, 0, 64, 1)
    assert lib.dt_state_importance(ctypes.byref(pw), None, None, None, None, None) == dt.DT_ERR_INVALID
    assert lib.dt_state_importance(ctypes.byref(pp), None, None, None, None, None) == dt.DT_ERR_INVALID
    assert lib.dt_state_importance(ctypes.byref(pp), 16 * 1024, 16 * 1024, 16 * 1024 + 4, None, None) == \
        dt.DT_ERR_UNSUPPORTED


def test_share_output_validated_on_the_host():
    import ctypes
    lib = dt.load()
    base = 1 << 20
    assert lib.dt_share_output(0, 1024, 64, None, None, None, None, None) == dt.DT_OK          # nothing to copy
    assert lib.dt_share_output(-1, 1024, 64, base, base, base, base, None) == dt.DT_ERR_INVALID
    assert lib.dt_share_output(2, 1024, 64, None, base, base, base, None) == dt.DT_ERR_INVALID
    # partially overlapping ranges are refused; identical ones are a no-op
    assert lib.dt_share_output(2, 1024, 64, base, base * 8, base + 4096, base * 16, None) == dt.DT_ERR_INVALID
    assert lib.dt_share_output(2, 1024, 64, base, base * 8, base, base * 8, None) == dt.DT_OK


def expected_partition_tiles(S, P, ks):
    """Partition-local 128-row tiles of the partitions of a key set, in order."""
    parts = orc.partitions(S, P)
    out = []
    for p in ks:
        a, b = parts[p]
        out += [(r, min(r + 128, b)) for r in range(a, b, 128)]
    return out


@pytest.mark.parametrize("S,P", [(1024, 4), (1000, 3), (5, 4), (2600, 64), (1800, 12), (32760, 16), (4097, 7),
                                 (300, 5), (129, 2), (100, 60), (640, 8)])
def test_key_set_tiles_match_oracle_key_sets(S, P):
    """The tiles the kernel visits for each (query tile, key set), from the
    same geometry code, cover exactly the oracle's key set: per partition,
    grouped (every group size), ungrouped."""
    for g in sorted({0, 1, 2, 3, 5, P}):
        p = dt.params(1, S, 64, P, dt.DT_MODE_ALL_COMPUTE, 0, 0, 1, g)
        nqt, nseg = dt.dt_plan_geometry(p)
        tiles = orc.query_tiles(S, P)
        for qt in range(0, nqt, max(1, nqt // 17)):
            sets = orc.key_sets_of_tile(tiles[qt][0], P, g)
            assert len(sets) == nseg
            for k in range(nseg):
                got = [(a, min(a + 128, e)) for a, e in dt.dt_key_set_tiles(p, qt, k)]
                assert got == expected_partition_tiles(S, P, sets[k]), (S, P, g, qt, k)


@pytest.mark.parametrize("S,W", [(16384, 1024), (1000, 100), (300, 64), (129, 1), (200, 400), (5000, 129)])
def test_window_key_set_tiles_by_brute_force(S, W):
    """Window mode: set 0 holds every key tile with a (query, key) pair inside
    the band, set 1 every key tile with a pair outside it (brute force over
    all pairs of the query tile)."""
    p = dt.params(1, S, 64, 1, dt.DT_MODE_WINDOW, 0, W, 1)
    nqt, _ = dt.dt_plan_geometry(p)
    keys = np.arange(S)
    for qt in range(0, nqt, max(1, nqt // 13)):
        rows = np.arange(qt * 128, min(qt * 128 + 128, S))
        inside = orc.window_in(rows, keys, W)
        want0, want1 = [], []
        for t in range(0, S, 128):
            blk = inside[:, t:t + 128]
            if blk.any():
                want0.append((t, min(t + 128, S)))
            if not blk.all():
                want1.append((t, min(t + 128, S)))
        got0 = sorted((a, min(a + 128, e)) for a, e in dt.dt_key_set_tiles(p, qt, 0))
        got1 = sorted((a, min(a + 128, e)) for a, e in dt.dt_key_set_tiles(p, qt, 1))
        assert got0 == want0 and got1 == want1, (S, W, qt)


def test_key_set_tiles_validated():
    import ctypes
    lib = dt.load()
    p = dt.params(1, 1024, 64, 4, dt.DT_MODE_ALL_COMPUTE, 0, 0, 1)
    for qt, k in ((-1, 0), (8, 0), (0, 4), (0, -1)):
        assert lib.dt_key_set_tiles(ctypes.byref(p), qt, k, None, None, 0) == dt.DT_ERR_INVALID
    assert lib.dt_key_set_tiles(ctypes.byref(p), 0, 0, None, None, 1) == dt.DT_ERR_INVALID
    assert lib.dt_key_set_tiles(ctypes.byref(p), 0, 0, None, None, 0) == 2


@pytest.mark.parametrize("wi", range(len(wl.WORKLOADS)))
def test_share_counts_match_oracle_counts(wi):
    """Attention sharing counts from libdt: across CFG branches half of the
    plan's computed blocks and FLOPs (the conditional half) with every other
    block skipped; across timesteps nothing computed and every block of every
    head skipped (the blocks an all-compute plan computes, by the oracle)."""
    w = wl.WORKLOADS[wi]
    H = 2 * w.H
    win = bool(w.window)
    mode = orc.MODE_WINDOW if win else orc.MODE_PROXIMITY
    P = 1 if win else w.P
    r = 0 if win else w.P // 2
    _, full, _ = orc.build_plan(orc.MODE_ALL_COMPUTE if not win else orc.MODE_WINDOW, H, w.S, w.D, P, 1,
                                window=w.window)
    p1 = dt.params(H, w.S, w.D, P, mode, r, w.window, 1)
    _, c1 = dt.dt_plan_build(p1)
    assert dt.dt_plan_share_counts(p1, dt.DT_SHARE_TIMESTEP) == {
        "computed_blocks": 0, "skipped_blocks": full["computed_blocks"] + full["skipped_blocks"], "computed_flops": 0}
    st = np.full(dt.dt_plan_geometry(p1), 1, dtype=np.int32)
    p2 = dt.params(H, w.S, w.D, P, mode, r, w.window, 2)
    _, c2 = dt.dt_plan_build(p2, st)
    for c in (c1, c2):
        _, ch, _ = orc.build_plan(mode, H // 2, w.S, w.D, P, 2 if c is c2 else 1, r=r, window=w.window,
                                  stamps=np.ones_like(st) if c is c2 else None)
        got = dt.dt_plan_share_counts(p1, dt.DT_SHARE_CFG, c)
        assert got["computed_blocks"] == ch["computed_blocks"]
        assert got["computed_flops"] == ch["computed_flops"]
        assert got["computed_blocks"] + got["skipped_blocks"] == c["computed_blocks"] + c["skipped_blocks"]


def test_share_calls_validated_on_the_host():
    import ctypes
    lib = dt.load()
    p = dt.params(3, 1024, 64, 4, dt.DT_MODE_PROXIMITY, 1, 0, 1)
    io = dt.Plan()
    assert lib.dt_plan_share_counts(ctypes.byref(p), dt.DT_SHARE_CFG, ctypes.byref(io)) == dt.DT_ERR_INVALID  # odd H
    p.H = 4
    assert lib.dt_plan_share_counts(ctypes.byref(p), 7, ctypes.byref(io)) == dt.DT_ERR_INVALID
    assert lib.dt_plan_share_counts(ctypes.byref(p), dt.DT_SHARE_CFG, None) == dt.DT_ERR_INVALID
    p.H = 3
    assert lib.dt_attn_cfg_shared(ctypes.byref(p), *([None] * 11), None) == dt.DT_ERR_INVALID
    p.H = 4
    assert lib.dt_attn_cfg_shared(ctypes.byref(p), *([None] * 11), None) == dt.DT_ERR_INVALID   # null buffers


def _sum_errors(err, plan, stamps_before):
    """(diff, norm) of the tracked pairs from the kernel's per-(head, warp)
    partial sums, added in the library's order (heads, then row groups) in
    float64; NaN where the pair has no previous state or was not computed."""
    nqt, nseg, H = err.shape[:3]
    diff = np.full((nqt, nseg), np.nan)
    norm = np.full((nqt, nseg), np.nan)
    for t in range(nqt):
        for k in range(nseg):
            if plan[t, k] != orc.COMPUTE or stamps_before[t, k] < 0:
                continue
            d = n = 0.0
            for h in range(H):
                for w in range(4):
                    d += float(err[t, k, h, w, 0])
                    n += float(err[t, k, h, w, 1])
            diff[t, k], norm[t, k] = d, n
    return diff, norm


@pytest.mark.parametrize("S,P,g,rho", [(4096, 16, 0, 0.5), (4096, 16, 4, 0.4), (1800, 12, 0, 0.3), (2600, 7, 2, 0.75),
                                        (777, 1, 0, 0.5), (3001, 5, 0, 1.0), (5000, 24, 5, 0.0), (650, 20, 3, 0.6)])
def test_anchor_planner_matches_oracle(S, P, g, rho):
    """dt_plan_build_anchor / dt_anchor_update against the oracle's
    anchor_plan / anchor_update on random measurements over 10 steps,
    including drift-triggered anchors: plans, anchor decisions and every
    piece of planner state bit-exact."""
    H, D = 3, 64
    p = dt.params(H, S, D, P, dt.DT_MODE_ANCHOR, 0, 0, 1, g)
    nqt, nseg = dt.dt_plan_geometry(p)
    theta = 0.05
    st_c, arr = dt.new_anchor_state(p, rho, theta)
    st_o = orc.AnchorState(nqt, nseg, rho, theta)
    stamps_c = np.full((nqt, nseg), -1, np.int32)
    stamps_o = stamps_c.copy()
    rng = np.random.Generator(np.random.PCG64(S + P + g))
    anchors = []
    for step in range(1, 11):
        p.step = step
        before = stamps_c.copy()
        plan_c, counts, anchored = dt.dt_plan_build_anchor(p, st_c, stamps_c)
        plan_o, anch_o = orc.anchor_plan(st_o, stamps_o, step, S, P, g)
        np.testing.assert_array_equal(plan_c, plan_o)
        assert anchored == anch_o
        anchors.append(anchored)
        stamps_o[plan_o == orc.COMPUTE] = step
        np.testing.assert_array_equal(stamps_c, stamps_o)
        # measurements: small drifts, a large one at step 5
        scale = 0.3 if step == 5 else 0.002
        err = np.empty((nqt, nseg, H, 4, 2), np.float32)
        err[..., 1] = rng.uniform(0.5, 2.0, (nqt, nseg, H, 4))
        err[..., 0] = (err[..., 1] * rng.uniform(0.0, scale, (nqt, nseg, H, 4)) ** 2).astype(np.float32)
        w_now = rng.uniform(0.0, 0.3, (nqt, nseg)).astype(np.float32) if anchored else None
        dt.dt_anchor_update(p, st_c, before, plan_c, err, w_now)
        diff, norm = _sum_errors(err, plan_c, before)
        orc.anchor_update(st_o, step, anchored, before, diff, norm, S, P, g, w_now=w_now)
        np.testing.assert_array_equal(arr["alpha"][:nqt], st_o.alpha)
        np.testing.assert_array_equal(arr["drift"][:nqt], st_o.drift)
        np.testing.assert_array_equal(arr["weights"][:nqt], st_o.w)
        assert np.float32(st_c.eps) == st_o.eps
    assert anchors[0] and anchors[5] and sum(anchors) >= 2      # the large drift of step 5 anchors step 6


def test_anchor_calls_validated():
    import ctypes
    lib = dt.load()
    p = dt.params(2, 1024, 64, 4, dt.DT_MODE_PROXIMITY, 1, 0, 1)
    st = dt.AnchorState()
    assert lib.dt_anchor_init(ctypes.byref(p), ctypes.byref(st)) == dt.DT_ERR_INVALID          # wrong mode, null arrays
    p.mode = dt.DT_MODE_ANCHOR
    assert lib.dt_anchor_init(ctypes.byref(p), ctypes.byref(st)) == dt.DT_ERR_INVALID          # null arrays
    st2, _ = dt.new_anchor_state(p, 0.5, 0.1)
    plan = dt.Plan()
    assert lib.dt_plan_build_anchor(ctypes.byref(p), ctypes.byref(st2), ctypes.byref(plan)) == dt.DT_ERR_INVALID
    st2.anchored = 1
    z = np.zeros(64, np.int32)
    assert lib.dt_anchor_update(ctypes.byref(p), ctypes.byref(st2), z.ctypes.data, z.ctypes.data, z.ctypes.data,
                                None) == dt.DT_ERR_INVALID                                       # anchor needs weights
    pw = dt.params(1, 1024, 64, 1, dt.DT_MODE_WINDOW, 0, 64, 1)
    assert lib.dt_attn_partial_fused_tracked(ctypes.byref(pw), *([None] * 11), 0, None) == dt.DT_ERR_INVALID
    assert lib.dt_plan_build(ctypes.byref(p), None, ctypes.byref(plan)) == dt.DT_ERR_INVALID      # needs its state


def test_plan_matches_oracle_on_random_geometry():
    """Seeded random geometries (ragged sequences, partition counts up to 24,
    groups of 1 to 5, every head dim), each through an anchor, two reuse steps
    with different r, an all-reuse step and an explicit plan: plans, counts
    and stamps bit-exact with the oracle's planner."""
    rng = np.random.Generator(np.random.PCG64(2024))
    for _ in range(40):
        S = int(rng.integers(1, 6000))
        P = int(rng.integers(1, 25))
        D = int(rng.choice([64, 72, 128]))
        H = int(rng.integers(1, 4))
        g = int(rng.choice([0, 0, 1, 2, 3, 5]))
        n_sets = P if g == 0 else -(-P // g)
        if n_sets + (1 if g else 0) > 64:
            continue
        p = dt.params(H, S, D, P, dt.DT_MODE_PROXIMITY, 0, 0, 1, g)
        nqt, nseg = dt.dt_plan_geometry(p)
        st = np.full((nqt, nseg), -1, np.int32)
        r1, r2 = (int(rng.integers(0, max(1, n_sets))) for _ in range(2))
        _, _, st = run_both(orc.MODE_PROXIMITY, H, S, D, P, 1, r=r1, stamps=st, group=g)
        _, _, st = run_both(orc.MODE_PROXIMITY, H, S, D, P, 2, r=r1, stamps=st, group=g)
        _, _, st = run_both(orc.MODE_PROXIMITY, H, S, D, P, 3, r=r2, stamps=st, group=g)
        _, _, st = run_both(orc.MODE_ALL_REUSE, H, S, D, P, 4, stamps=st, group=g)
        ex = (rng.random((nqt, nseg)) < 0.5).astype(np.uint8)
        run_both(orc.MODE_EXPLICIT, H, S, D, P, 5, stamps=st, explicit=ex, group=g)


def test_window_plan_matches_oracle_on_random_geometry():
    rng = np.random.Generator(np.random.PCG64(2025))
    for _ in range(30):
        S = int(rng.integers(1, 9000))
        W = int(rng.integers(1, 2 * S + 2))
        H, D = int(rng.integers(1, 4)), int(rng.choice([64, 72, 128]))
        p = dt.params(H, S, D, 1, dt.DT_MODE_WINDOW, 0, W, 1)
        nqt, nseg = dt.dt_plan_geometry(p)
        st = np.full((nqt, nseg), -1, np.int32)
        for step in (1, 2, 3):
            _, _, st = run_both(orc.MODE_WINDOW, H, S, D, 1, step, window=W, stamps=st)


def test_plan_parameters_fuzzed():
    """Seeded random parameter sets, valid and invalid (negative, zero, huge
    or inconsistent fields, every mode): the host planner either rejects them
    with a status code or builds a plan whose counts add up, and never
    crashes; accepted all-compute plans match the oracle's."""
    import ctypes
    lib = dt.load()
    rng = np.random.Generator(np.random.PCG64(77))
    pick = lambda *vals: int(rng.choice(vals))
    accepted = 0
    for _ in range(400):
        H = pick(-1, 0, 1, 2, 3, 1 << 20)
        S = pick(-5, 0, 1, 127, 128, 129, 1000, 4097, 1 << 30)
        D = pick(0, 8, 64, 72, 100, 128, 256)
        P = pick(-1, 0, 1, 3, 16, 64, 65, 200)
        mode = pick(-1, 0, 1, 2, 3, 4, 5, 6, 7, 99)
        r = pick(-2, 0, 1, 7, 15, 64)
        window = pick(-1, 0, 1, 64, 1000, 1 << 30)
        step = pick(-1, 0, 1, 2, 5)
        group = pick(-1, 0, 1, 3, 8, 100)
        p = dt.params(H, S, D, P, mode, r, window, step, group)
        nqt, nseg = ctypes.c_int32(), ctypes.c_int32()
        rc = lib.dt_plan_geometry(ctypes.byref(p), ctypes.byref(nqt), ctypes.byref(nseg))
        if rc != dt.DT_OK:
            assert rc in (dt.DT_ERR_INVALID, dt.DT_ERR_UNSUPPORTED), rc
            continue
        if nqt.value * nseg.value > 1 << 22:                 # huge but valid: skip the build
            continue
        plan = np.zeros((max(nqt.value, 1), max(nseg.value, 1)), np.uint8)
        st = np.full(plan.shape, 1, np.int32)                # every slot cached at step 1
        out = dt.Plan()
        out.plan = plan.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))
        out.stamps = st.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
        ex = np.zeros(plan.shape, np.uint8)
        rc = lib.dt_plan_build(ctypes.byref(p), ex.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)), ctypes.byref(out))
        if rc != dt.DT_OK:
            assert rc in (dt.DT_ERR_INVALID, dt.DT_ERR_UNSUPPORTED, dt.DT_ERR_CACHE_EMPTY), rc
            continue
        accepted += 1
        assert out.computed_blocks >= 0 and out.skipped_blocks >= 0
        assert set(np.unique(plan[: nqt.value, : nseg.value])) <= {0, 1}
        if mode == dt.DT_MODE_ALL_COMPUTE and group == 0 and H * S < 1 << 16:
            want, counts, _ = orc.build_plan(orc.MODE_ALL_COMPUTE, H, S, D, P, step)
            np.testing.assert_array_equal(plan[: nqt.value, : nseg.value], want)
            assert out.computed_blocks == counts["computed_blocks"]
    assert accepted > 20
