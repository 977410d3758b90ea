"""GPU parity: the fused CUDA path against the float64 oracle on the same
seeded bf16 inputs, through the C ABI.

Small workloads are compared element by element; the full-size ones (in the
launch configuration the benchmark times) on sampled heads and rows, which
the oracle follows exactly through the whole schedule (rows are independent).
"""

import numpy as np
import pytest
import torch

import oracle as orc
import partitioned_attention_state_b200 as dt
from partitioned_attention_state_b200 import workloads as wl
from partitioned_attention_state_b200.session import Session

from parity import check_lse, check_out, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dt.dt_set_wait_limit_ns(2_000_000_000)
    yield
    torch.cuda.synchronize()


def run_partition_schedule(H, S, D, P, schedule, inputs, heads=None, rows=None, check_untouched=False,
                           output_scaled=False, group=0, sess=None, cache=None, state_dtype=0):
    """schedule: list of (step, mode, r, explicit); inputs: callable -> (q,k,v) bits.
    group > 0: grouped key sets (one cache slot per group).  A session and
    oracle cache may be passed in to continue an earlier schedule."""
    if sess is None:
        sess = Session(H, S, D, P, mode=dt.DT_MODE_PROXIMITY, group=group, state_dtype=state_dtype)
        cache = orc.StateCache(bf16=state_dtype == dt.DT_STATE_BF16)
    group = sess.group
    hs = list(range(H)) if heads is None else list(heads)
    rs = np.arange(S) if rows is None else np.asarray(rows)
    for step, mode, r, explicit in schedule:
        q, k, v = inputs()
        sess.set_inputs(q, k, v)
        sess.r = r
        sess.counters.zero_()
        before = None
        if check_untouched:
            before = (sess.cache_O.clone(), sess.cache_L.clone())
        counts = sess.step(step, mode=mode, explicit=explicit)
        sess.check()
        plan = sess.last_plan
        # device counters equal the host plan counts (bit-exact)
        c = sess.counters.cpu().numpy()
        assert int(c[0]) == counts["computed_blocks"] and int(c[1]) == counts["skipped_blocks"]
        assert int(c[2]) == H * int((plan == 1).sum()) and int(c[3]) == H * int((plan == 0).sum())
        Q, K, V = (orc.widen_bf16(x[hs]) for x in (q, k, v))
        O_ref, L_ref, fresh = orc.partition_step(Q, K, V, plan, S, P, cache, rows=rs, group=group)
        O_gpu = to_np(sess.O[hs][:, rs])
        L_gpu = to_np(sess.L[hs][:, rs])
        check_out(O_gpu, O_ref, f"O step {step}", output_scaled=output_scaled)
        check_lse(L_gpu, L_ref, f"LSE step {step}")
        # fresh states written to their slots
        co, cl = sess.cache_O, sess.cache_L
        for (kk, hi), items in fresh.items():
            h = hs[hi]
            for rr, (o_f, l_f) in items:
                check_out(to_np(co[kk, h][rr]), o_f, f"cache OUT k={kk} h={h} step {step}",
                          output_scaled=output_scaled)
                check_lse(to_np(cl[kk, h][rr]), l_f, f"cache LSE k={kk} h={h} step {step}")
        if before is not None:
            tiles = orc.query_tiles(S, P)
            for t, (_, q0, q1) in enumerate(tiles):
                for kk in range(sess.nseg):
                    if plan[t, kk] == orc.REUSE:
                        assert torch.equal(before[0][kk, :, q0:q1], co[kk, :, q0:q1])
                        assert torch.equal(before[1][kk, :, q0:q1], cl[kk, :, q0:q1])
    return sess, cache


def proximity_schedule(steps, r):
    return [(t, dt.DT_MODE_PROXIMITY, r, None) for t in range(1, steps + 1)]


def stream_of(H, S, D, sigma, seed=0):
    s = wl.InputStream(H, S, D, sigma, seed=seed)
    return s.next_step


# ----------------------------------------------------------------- workloads

def test_tiny_workload_full_parity():
    w = wl.WORKLOADS[0]
    run_partition_schedule(w.H, w.S, w.D, w.P, proximity_schedule(w.steps, w.reuse[0]), wl.stream_for(w).next_step,
                           check_untouched=True)


@pytest.mark.parametrize("r", wl.WORKLOADS[1].reuse)
def test_dit_xl2_workload_full_parity(r):
    w = wl.WORKLOADS[1]
    run_partition_schedule(w.H, w.S, w.D, w.P, proximity_schedule(w.steps, r), wl.stream_for(w).next_step,
                           check_untouched=True)


def sample_rows(S, P, n_extra=40, seed=0):
    """Rows at tile and partition edges plus random ones."""
    rows = set()
    for _, q0, q1 in orc.query_tiles(S, P):
        rows.update((q0, q1 - 1))
    rng = np.random.Generator(np.random.PCG64(seed))
    rows.update(rng.choice(S, size=n_extra, replace=False).tolist())
    rows = sorted(rows)
    if len(rows) > 160:
        keep = set(rng.choice(len(rows), size=160, replace=False).tolist())
        rows = [r for i, r in enumerate(rows) if i in keep or r in (0, S - 1)]
    return np.array(sorted(set(rows)))


def test_pixart_workload_sampled_rows():
    w = wl.WORKLOADS[2]
    run_partition_schedule(w.H, w.S, w.D, w.P, proximity_schedule(2, w.reuse[0]), wl.stream_for(w).next_step,
                           heads=[0, 7, 15], rows=sample_rows(w.S, w.P))


def test_video_workload_full_size_sampled_rows():
    """Full-size 3D video workload in the benchmark's launch configuration:
    anchor step, then reuse steps at 25% and 75%."""
    w = wl.WORKLOADS[3]
    sched = [(1, dt.DT_MODE_PROXIMITY, 4, None), (2, dt.DT_MODE_PROXIMITY, 4, None),
             (3, dt.DT_MODE_PROXIMITY, 12, None)]
    run_partition_schedule(w.H, w.S, w.D, w.P, sched, wl.stream_for(w).next_step, heads=[0, 39],
                           rows=sample_rows(w.S, w.P, n_extra=24))



def test_video_workload_benchmark_configuration():
    """The configuration bench.py times: the full-size video workload, an
    anchor step, then two 50%-reuse steps (8 of 16 partitions reused), on
    sampled heads and rows, including the fresh cache slots."""
    w = wl.WORKLOADS[3]
    sched = [(1, dt.DT_MODE_PROXIMITY, 8, None), (2, dt.DT_MODE_PROXIMITY, 8, None),
             (3, dt.DT_MODE_PROXIMITY, 8, None)]
    run_partition_schedule(w.H, w.S, w.D, w.P, sched, wl.stream_for(w).next_step, heads=[0, 21, 39],
                           rows=sample_rows(w.S, w.P, n_extra=24))

# ------------------------------------------------------------------ edge cases

@pytest.mark.parametrize("H,S,D,P,r", [
    (2, 1000, 72, 3, 1),      # ragged partitions and tiles
    (1, 5, 64, 4, 2),         # tiny sequence, one empty partition
    (2, 300, 128, 5, 2),      # D=128, short partitions (1 ragged tile each)
    (3, 2000, 64, 7, 3),
    (1, 128, 72, 1, 0),       # one tile, one partition
    (2, 4100, 128, 2, 1),     # 33 key tiles per head, ragged tail of 4 rows
    (1, 2600, 64, 64, 40),    # the most partitions the fused kernel takes (64-bit plan mask)
    (1, 1800, 72, 12, 5),     # P not a multiple of 4: byte-wise plan rows
])
def test_ragged_geometry(H, S, D, P, r):
    run_partition_schedule(H, S, D, P, proximity_schedule(3, r), stream_of(H, S, D, 0.05, seed=S),
                           check_untouched=True)


@pytest.mark.parametrize("kind", ["unit", "spiky"])
@pytest.mark.parametrize("D", [64, 72, 128])
def test_stress_inputs(kind, D):
    H, S, P = 2, 700, 3
    q, k, v = wl.stress_inputs(H, S, D, kind, seed=D)
    run_partition_schedule(H, S, D, P, [(1, dt.DT_MODE_ALL_COMPUTE, 0, None)], lambda: (q, k, v),
                           output_scaled=True)


def perturbed(bits, sigma, seed):
    """bf16 inputs plus sigma * N(0,1), rounded back to bf16 (a later step of
    a stress set)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = wl.bf16_bits_to_f32(bits) + np.float32(sigma) * rng.standard_normal(bits.shape, dtype=np.float32)
    return wl.f32_to_bf16_bits(x)


@pytest.mark.parametrize("kind", ["unit", "spiky"])
@pytest.mark.parametrize("D,g", [(64, 0), (72, 0), (128, 0), (128, 2)])
def test_stress_inputs_through_reuse(kind, D, g):
    """Stress sets through an anchor and then reuse steps: cached states with
    a large spread of LSEs (logits above 20 in "spiky") are composed with
    fresh ones by the epilogue's reuse merge."""
    H, S, P = 2, 1500, 6
    q, k, v = wl.stress_inputs(H, S, D, kind, seed=D + 1)
    steps = [(q, k, v)] + [tuple(perturbed(x, 0.05, 10 * t + j) for j, x in enumerate((q, k, v))) for t in (1, 2)]
    it = iter(steps)
    sched = [(1, dt.DT_MODE_PROXIMITY, 2, None), (2, dt.DT_MODE_PROXIMITY, 2, None),
             (3, dt.DT_MODE_PROXIMITY, 1 if g else 4, None)]
    run_partition_schedule(H, S, D, P, sched, lambda: next(it), output_scaled=True, group=g, check_untouched=True)


def test_all_reuse_reproduces_previous_output_and_explicit_plan():
    H, S, D, P = 2, 900, 72, 4
    q, k, v = wl.InputStream(H, S, D, 0.0, seed=5).next_step()
    sched = [(1, dt.DT_MODE_ALL_COMPUTE, 0, None), (2, dt.DT_MODE_ALL_REUSE, 0, None)]
    nqt = len(orc.query_tiles(S, P))
    ex = (np.arange(nqt * P).reshape(nqt, P) % 2).astype(np.uint8)
    sched.append((3, dt.DT_MODE_EXPLICIT, 0, ex))
    sess, _ = run_partition_schedule(H, S, D, P, sched, lambda: (q, k, v))
    # with unchanged inputs every plan gives full attention
    full, lf = orc.attention_state(orc.widen_bf16(q[1]), orc.widen_bf16(k[1]), orc.widen_bf16(v[1]),
                                   orc.softmax_scale(D))
    check_out(to_np(sess.O[1]), full)
    check_lse(to_np(sess.L[1]), lf)


def test_output_guard_bands_untouched():
    H, S, D, P = 2, 640, 64, 4
    sess = Session(H, S, D, P, mode=dt.DT_MODE_PROXIMITY)
    pad = 4096
    big_o = torch.full((H * S * D + 2 * pad,), 7.0, dtype=torch.bfloat16, device="cuda")
    big_l = torch.full((H * S + 2 * pad,), 7.0, dtype=torch.float32, device="cuda")
    sess.O = big_o[pad:pad + H * S * D].view(H, S, D)
    sess.L = big_l[pad:pad + H * S].view(H, S)
    sess.set_inputs(*wl.InputStream(H, S, D, 0.05, seed=9).next_step())
    sess.step(1)
    sess.check()
    for t in (big_o[:pad], big_o[-pad:], big_l[:pad], big_l[-pad:]):
        assert torch.all(t == 7.0)
    assert torch.isfinite(sess.O.float()).all()


@pytest.mark.parametrize("D", [72, 128])
def test_cache_alignment_16_matches_32(D):
    """A state cache that starts on a 16-byte (not 32-byte) boundary takes
    the 16-byte store path for fresh states; outputs, LSEs and every cache
    byte equal those of a 32-byte-aligned cache."""
    H, S, P = 2, 1100, 4
    q, k, v = wl.InputStream(H, S, D, 0.05, seed=21).next_step()
    q2, k2, v2 = wl.InputStream(H, S, D, 0.05, seed=22).next_step()
    runs = []
    for offset in (0, 4):                          # floats: 0 or 16 bytes past a 256-byte boundary
        sess = Session(H, S, D, P, mode=dt.DT_MODE_PROXIMITY, reuse_per_row=2)
        n = sess.cache_O.numel()
        big = torch.zeros(n + 8, dtype=torch.float32, device="cuda")
        sess.cache_O = big[offset:offset + n].view(sess.cache_O.shape)
        assert (sess.cache_O.data_ptr() % 32 == 0) == (offset == 0)
        sess.set_inputs(q, k, v)
        sess.step(1)
        sess.set_inputs(q2, k2, v2)
        sess.step(2)
        sess.check()
        runs.append((sess.O.clone(), sess.L.clone(), sess.cache_O.clone(), sess.cache_L.clone()))
    for a, b in zip(*runs):
        assert torch.equal(a.view(torch.int32) if a.dtype == torch.float32 else a.view(torch.int16),
                           b.view(torch.int32) if b.dtype == torch.float32 else b.view(torch.int16))


# ------------------------------------------------------------------ window mode

def run_window_schedule(H, S, D, W, steps, inputs, heads=None, rows=None):
    sess = Session(H, S, D, 1, mode=dt.DT_MODE_WINDOW, window=W)
    R = {}
    hs = list(range(H)) if heads is None else list(heads)
    rs = np.arange(S) if rows is None else np.asarray(rows)
    for step in range(1, steps + 1):
        q, k, v = inputs()
        sess.set_inputs(q, k, v)
        sess.counters.zero_()
        counts = sess.step(step)
        sess.check()
        c = sess.counters.cpu().numpy()
        assert int(c[0]) == counts["computed_blocks"] and int(c[1]) == counts["skipped_blocks"]
        Q, K, V = (orc.widen_bf16(x[hs]) for x in (q, k, v))
        O_ref, L_ref = orc.window_step(Q, K, V, W, step == 1, R, rows=rs)
        check_out(to_np(sess.O[hs][:, rs]), O_ref, f"O step {step}")
        check_lse(to_np(sess.L[hs][:, rs]), L_ref, f"LSE step {step}")
        if step == 1:
            R_ref = np.stack([np.stack([R[(hi, int(r))] for r in rs]) for hi in range(len(hs))])
            check_out(to_np(sess.R[hs][:, rs]), R_ref, "R", max_abs=1e-2, rel=1e-2)
    return sess


@pytest.mark.parametrize("H,S,D,W", [(2, 1000, 72, 100), (1, 300, 64, 64), (2, 200, 128, 400), (1, 129, 72, 1),
                                     (2, 2048, 72, 1024), (1, 5000, 64, 129)])
def test_window_small(H, S, D, W):
    run_window_schedule(H, S, D, W, 3, stream_of(H, S, D, 0.03, seed=W))


def test_window_workload_full_size_sampled_rows():
    """The full-size window workload over its whole schedule: the anchor step
    (full attention, R made) and the three window + residual steps."""
    w = wl.WORKLOADS[4]
    rows = np.unique(np.concatenate([np.arange(0, 130), np.arange(w.S - 130, w.S),
                                     np.random.Generator(np.random.PCG64(3)).choice(w.S, 60, replace=False)]))
    run_window_schedule(w.H, w.S, w.D, w.window, w.steps, wl.stream_for(w).next_step, heads=[0, 15], rows=rows)


def run_window_abi(H, S, D, W, steps, inputs, fill=float("nan")):
    """Window mode through the C ABI directly, with caller buffers that start
    filled with `fill` (NaN by default): every row of R must be written at the
    anchor step, whatever the caller's buffer held."""
    dev = "cuda"
    R = torch.full((H, S, D), fill, dtype=torch.float32, device=dev)
    O = torch.full((H, S, D), fill, dtype=torch.bfloat16, device=dev)
    L = torch.full((H, S), fill, dtype=torch.float32, device=dev)
    Qd, Kd, Vd = (torch.empty((H, S, D), dtype=torch.bfloat16, device=dev) for _ in range(3))
    counters = torch.zeros(4, dtype=torch.int64, device=dev)
    status = torch.zeros(4, dtype=torch.int32, device=dev)
    Rref = {}
    stamps = None
    for step in range(1, steps + 1):
        q, k, v = inputs()
        for dst, src in ((Qd, q), (Kd, k), (Vd, v)):
            dst.copy_(torch.from_numpy(src.view(np.int16)).view(torch.bfloat16))
        p = dt.params(H, S, D, 1, dt.DT_MODE_WINDOW, 0, W, step)
        if stamps is None:
            stamps = np.full(dt.dt_plan_geometry(p), -1, dtype=np.int32)
        plan, counts = dt.dt_plan_build(p, stamps)
        d_plan = torch.from_numpy(plan).to(dev)
        counters.zero_()
        dt.dt_attn_partial_fused(p, d_plan, Qd, Kd, Vd, None, None, R, O, L, counters, status)
        torch.cuda.synchronize()
        assert int(status[0]) == 0, dt.dt_status_string(int(status[0]))
        c = counters.cpu().numpy()
        assert int(c[0]) == counts["computed_blocks"] and int(c[1]) == counts["skipped_blocks"]
        O_ref, L_ref = orc.window_step(q, k, v, W, step == 1, Rref)
        if step == 1:
            R_ref = np.stack([np.stack([Rref[(h, r)] for r in range(S)]) for h in range(H)])
            check_out(to_np(R), R_ref, "R", max_abs=1e-2, rel=1e-2)
        check_out(to_np(O), O_ref, f"O step {step}")
        check_lse(to_np(L), L_ref, f"LSE step {step}")


@pytest.mark.parametrize("H,S,D,W", [
    (2, 200, 128, 400),      # W >= 2S: every key in every window, R = 0 everywhere
    (1, 2000, 72, 1900),     # interior query tiles whose band covers all keys (empty complement)
    (1, 2000, 64, 1900),
    (2, 1000, 128, 100),     # ordinary band: every row has a complement
])
def test_window_residual_written_for_every_row(H, S, D, W):
    run_window_abi(H, S, D, W, 3, stream_of(H, S, D, 0.03, seed=S + W))


@pytest.mark.parametrize("D", [72, 128])
def test_window_spiky_inputs(D):
    """Window mode on the spiky stress set: the residual of rows whose large
    logits fall outside the band is large, and later steps add it back."""
    H, S, W = 2, 1200, 256
    q, k, v = wl.stress_inputs(H, S, D, "spiky", seed=D + 5)
    steps = iter([(q, k, v)] + [tuple(perturbed(x, 0.05, 20 * t + j) for j, x in enumerate((q, k, v)))
                                for t in (1, 2)])
    sess = Session(H, S, D, 1, mode=dt.DT_MODE_WINDOW, window=W)
    sess.R.fill_(float("nan"))
    R = {}
    for step in (1, 2, 3):
        qq, kk, vv = next(steps)
        sess.set_inputs(qq, kk, vv)
        sess.step(step)
        sess.check()
        O_ref, L_ref = orc.window_step(qq, kk, vv, W, step == 1, R)
        check_out(to_np(sess.O), O_ref, f"O step {step}", output_scaled=True)
        check_lse(to_np(sess.L), L_ref, f"LSE step {step}")


@pytest.mark.gpu
def test_graph_replay_matches_eager_step():
    """A step replayed from a captured CUDA graph writes the same bytes as the
    eager step (same kernel, same inputs, same plan)."""
    w = wl.BY_NAME["dit_xl2_512_32x32_h16_d72_p8"]
    sess = Session(w.H, w.S, w.D, w.P, reuse_per_row=4)
    s = wl.stream_for(w)
    sess.set_inputs(*s.next_step())
    sess.step(1)
    sess.set_inputs(*s.next_step())
    cache_O, cache_L = sess.cache_O.clone(), sess.cache_L.clone()
    counts = sess.step(2)
    sess.check()
    o_eager, l_eager = sess.O.clone(), sess.L.clone()
    sess.cache_O.copy_(cache_O)
    sess.cache_L.copy_(cache_L)
    sess.O.zero_()
    sess.L.zero_()
    g = sess.capture_step(2)
    for _ in range(3):
        assert g.replay() == counts
    sess.check()
    assert torch.equal(sess.O.view(torch.int16), o_eager.view(torch.int16))
    assert torch.equal(sess.L, l_eager)


def _pinned_like(t, dtype=None):
    return torch.empty(t.shape, dtype=t.dtype if dtype is None else dtype).pin_memory()


@pytest.mark.gpu
@pytest.mark.parametrize("name,groups", [("dit_xl2_512_32x32_h16_d72_p8", 3), ("tiny_4x16x16_h2_d64_p4", 8),
                                         ("dit_xl2_512_32x32_h16_d72_p8", 1)])
def test_host_step_head_groups_match_whole_step(name, groups):
    """Session.step_host (head-range launches pipelined with their copies)
    writes the same bytes as the whole-step launch: same outputs, same cache
    slots, same counters."""
    w = wl.BY_NAME[name]
    s = wl.stream_for(w)
    steps = [s.next_step() for _ in range(3)]
    a = Session(w.H, w.S, w.D, w.P, reuse_per_row=w.P // 2)
    b = Session(w.H, w.S, w.D, w.P, reuse_per_row=w.P // 2)
    ho = _pinned_like(b.O, torch.int16)
    hl = _pinned_like(b.L)
    for t, (q, k, v) in enumerate(steps, start=1):
        a.set_inputs(q, k, v)
        a.counters.zero_()
        ca = a.step(t)
        a.check()
        hq = [torch.from_numpy(x.view(np.int16)).pin_memory() for x in (q, k, v)]
        b.counters.zero_()
        cb = b.step_host(t, *hq, ho, hl, groups=groups)
        torch.cuda.current_stream().synchronize()
        b.check()
        assert ca == cb
        assert torch.equal(a.counters, b.counters)
        assert torch.equal(a.O.view(torch.int16).cpu(), ho)
        assert torch.equal(a.L.cpu(), hl)
        assert torch.equal(a.cache_O, b.cache_O) and torch.equal(a.cache_L, b.cache_L)


@pytest.mark.gpu
def test_host_step_window_mode_matches_whole_step():
    """Window mode through step_host: anchor step (writes R) and two residual
    steps, byte-identical to whole-step launches."""
    w = wl.BY_NAME["window_128x128_h16_d72_w1024"]
    H, S = 4, 4096
    s = wl.InputStream(H, S, w.D, w.sigma, seed=3)
    a = Session(H, S, w.D, mode=dt.DT_MODE_WINDOW, window=w.window)
    b = Session(H, S, w.D, mode=dt.DT_MODE_WINDOW, window=w.window)
    ho = _pinned_like(b.O, torch.int16)
    hl = _pinned_like(b.L)
    for t in (1, 2, 3):
        q, k, v = s.next_step()
        a.set_inputs(q, k, v)
        a.step(t)
        a.check()
        hq = [torch.from_numpy(x.view(np.int16)).pin_memory() for x in (q, k, v)]
        b.step_host(t, *hq, ho, hl, groups=3)
        torch.cuda.current_stream().synchronize()
        b.check()
        assert torch.equal(a.O.view(torch.int16).cpu(), ho)
        assert torch.equal(a.L.cpu(), hl)
        assert torch.equal(a.R, b.R)



# ------------------------------------------------------------ state grouping

@pytest.mark.parametrize("H,S,D,P,g,rs", [
    (16, 1024, 72, 8, 2, (1, 2, 3)),     # DiT-XL/2-like geometry, groups of 2
    (2, 1024, 64, 4, 2, (1, 2)),         # the Fig. 6 layout (CP = 4, groups of 2)
    (2, 2048, 128, 16, 4, (2, 1, 3)),    # the video grouping on a short sequence
    (1, 2600, 64, 64, 8, (3, 7)),        # 1 + 8 key sets, 41-row partitions (one short tile each)
    (2, 1800, 72, 12, 5, (1, 2)),        # last group short, 150-row partitions (ragged tiles)
    (1, 1000, 128, 7, 3, (2,)),          # P not a multiple of g, ragged last partition
    (2, 1024, 72, 8, 1, (3, 7)),         # groups of one: 1 + P key sets, the local group empty
])
def test_grouped_schedule_parity(H, S, D, P, g, rs):
    sched = [(1, dt.DT_MODE_PROXIMITY, rs[0], None)] + \
            [(t + 2, dt.DT_MODE_PROXIMITY, r, None) for t, r in enumerate(rs)]
    run_partition_schedule(H, S, D, P, sched, stream_of(H, S, D, 0.05, seed=S + g), check_untouched=True, group=g)


def test_grouped_video_full_size_sampled_rows():
    """The video workload with groups of 4 partitions (1 + 4 key sets) in the
    benchmark's launch configuration: anchor, then 2 of 4 groups reused."""
    w = wl.WORKLOADS[3]
    sched = [(1, dt.DT_MODE_PROXIMITY, 2, None), (2, dt.DT_MODE_PROXIMITY, 2, None),
             (3, dt.DT_MODE_PROXIMITY, 3, None)]
    run_partition_schedule(w.H, w.S, w.D, w.P, sched, wl.stream_for(w).next_step, heads=[0, 39],
                           rows=sample_rows(w.S, w.P, n_extra=24), group=4)


# m = ceil(P / g) old groups: 4, 8 and 16 take the row-at-once kernel, 20 the group-by-group one
@pytest.mark.parametrize("P,g,f", [(8, 1, 2), (16, 2, 2), (12, 1, 3), (7, 2, 4), (12, 1, 5), (16, 1, 8), (20, 1, 2)])
def test_group_compose_matches_oracle(P, g, f):
    """Dynamic Group State Compose on the GPU: the regrouped cache equals the
    oracle's N-way composition of the GPU's own cached states (fp32 rounding
    only), the stamps equal the oracle's, and later steps on the coarse
    layout match the oracle run through the same regrouping."""
    H, S, D = 2, 128 * P + 40, 64
    s = stream_of(H, S, D, 0.05, seed=P * 10 + g)
    sess, cache = run_partition_schedule(H, S, D, P, [(1, dt.DT_MODE_PROXIMITY, 1, None),
                                                      (2, dt.DT_MODE_PROXIMITY, 1, None)], s, group=g)
    m = -(-P // g)
    before_O = to_np(sess.cache_O[: 1 + m])
    before_L = to_np(sess.cache_L[: 1 + m])
    st_before = sess.stamps.copy()
    sess.compose_groups(f)
    sess.check()
    m2 = -(-m // f)
    assert sess.group == g * f and sess.nseg == 1 + m2
    new_cache, st_want = orc.compose_groups(cache, st_before, P, g, f, list(range(H)), np.arange(S), S, D)
    np.testing.assert_array_equal(sess.stamps, st_want)
    np.testing.assert_array_equal(to_np(sess.cache_O[0]), before_O[0])
    for i in range(m2):
        js = range(f * i, min(f * i + f, m))
        want_o, want_l = orc.compose_n([(before_O[1 + j].reshape(-1, D), before_L[1 + j].reshape(-1)) for j in js])
        got_o = to_np(sess.cache_O[1 + i]).reshape(-1, D)
        got_l = to_np(sess.cache_L[1 + i]).reshape(-1)
        np.testing.assert_allclose(got_o, want_o, rtol=2e-5, atol=2e-6)
        np.testing.assert_allclose(got_l, want_l, rtol=0, atol=2e-5)
    run_partition_schedule(H, S, D, P, [(3, dt.DT_MODE_PROXIMITY, 1, None), (4, dt.DT_MODE_ALL_REUSE, 0, None)], s,
                           sess=sess, cache=new_cache)



# ------------------------------------------------------------ bf16 state cache

@pytest.mark.parametrize("H,S,D,P,g,rs", [
    (16, 1024, 72, 8, 0, (4, 2, 6)),     # DiT-XL/2-like geometry
    (2, 1024, 64, 4, 0, (2, 1)),
    (2, 2600, 128, 7, 0, (3, 5)),        # D = 128, ragged partitions
    (2, 2048, 128, 16, 4, (2, 1, 3)),    # with grouping
    (1, 1800, 72, 12, 5, (1, 2)),
])
def test_bf16_state_cache_schedule_parity(H, S, D, P, g, rs):
    """The bf16 state cache: fresh states are stored rounded to bf16 and
    reused from there; outputs, cached states and untouched slots match the
    oracle run with the same rounding of its cache."""
    sched = [(1, dt.DT_MODE_PROXIMITY, rs[0], None)] + \
            [(t + 2, dt.DT_MODE_PROXIMITY, r, None) for t, r in enumerate(rs)]
    sess, _ = run_partition_schedule(H, S, D, P, sched, stream_of(H, S, D, 0.05, seed=S + 7), check_untouched=True,
                                     group=g, state_dtype=dt.DT_STATE_BF16)
    assert sess.cache_O.dtype == torch.bfloat16


def test_bf16_state_cache_video_full_size_sampled_rows():
    w = wl.WORKLOADS[3]
    sched = [(1, dt.DT_MODE_PROXIMITY, 8, None), (2, dt.DT_MODE_PROXIMITY, 8, None)]
    run_partition_schedule(w.H, w.S, w.D, w.P, sched, wl.stream_for(w).next_step, heads=[0, 39],
                           rows=sample_rows(w.S, w.P, n_extra=16), state_dtype=dt.DT_STATE_BF16)


# ------------------------------------------------------ partition importance

@pytest.mark.parametrize("H,S,D,P,g", [(2, 1024, 64, 4, 0), (2, 2048, 128, 16, 4), (3, 1800, 72, 12, 5),
                                       (2, 2600, 64, 7, 0)])
def test_importance_weights_and_plan_match_oracle(H, S, D, P, g):
    """dt_state_importance after an anchor equals the oracle's importance of
    the same inputs, the weights of a row sum to one, and importance-planned
    steps use the oracle's rule on those weights and match it in output."""
    s = wl.InputStream(H, S, D, 0.05, seed=S + P)
    inputs = [s.next_step() for _ in range(3)]
    it = iter(inputs)
    sess, cache = run_partition_schedule(H, S, D, P, [(1, dt.DT_MODE_PROXIMITY, 0, None)], lambda: next(it),
                                         group=g)
    w_gpu = sess.measure_importance()
    assert w_gpu.shape == (sess.nqt, sess.nseg) and w_gpu.dtype == np.float32
    np.testing.assert_allclose(w_gpu.sum(axis=1), 1.0, rtol=0, atol=1e-4)
    q, k, v = inputs[0]
    oc = orc.StateCache()
    plan1, _, _ = orc.build_plan(orc.MODE_ALL_COMPUTE, H, S, D, P, step=1, group=g)
    _, L, _ = orc.partition_step(q, k, v, plan1, S, P, oc, group=g)
    Lmap = {(h, r): float(L[h, r]) for h in range(H) for r in range(S)}
    w_ref = orc.state_importance(oc, Lmap, S, P, g, range(H), sess.nseg)
    np.testing.assert_allclose(w_gpu, w_ref, rtol=0, atol=2e-3)
    for step in (2, 3):
        want, _, _ = orc.build_plan(orc.MODE_IMPORTANCE, H, S, D, P, step, r=2, stamps=sess.stamps.copy(), group=g,
                                    weights=w_gpu)
        run_partition_schedule(H, S, D, P, [(step, dt.DT_MODE_IMPORTANCE, 2, None)], lambda: next(it),
                               check_untouched=True, sess=sess, cache=cache)
        np.testing.assert_array_equal(sess.last_plan, want)


# ------------------------------------------------------- attention sharing

@pytest.mark.parametrize("g,sd", [(0, 0), (2, 0), (0, 1)])
def test_cfg_shared_step(g, sd):
    """Sharing across CFG branches: heads [0, H/2) (conditional) are computed
    and match the oracle on their own inputs; heads [H/2, H) receive the same
    output bytes, their inputs are ignored, and the states the conditional
    heads computed become theirs too (same cache bytes).  A later ordinary
    step on both halves then reuses those states and matches the oracle on
    every head."""
    Hb, S, D, P = 2, 1024, 64, 4
    r = 1
    cond = wl.InputStream(Hb, S, D, 0.05, seed=90)
    other = wl.InputStream(Hb, S, D, 0.5, seed=91)
    sess = Session(2 * Hb, S, D, P, reuse_per_row=r, group=g, state_dtype=sd)
    cache = orc.StateCache(bf16=sd == dt.DT_STATE_BF16)
    for step in (1, 2):
        qc, kc, vc = cond.next_step()
        qu, ku, vu = other.next_step()
        sess.set_inputs(*(np.concatenate([a, b]) for a, b in ((qc, qu), (kc, ku), (vc, vu))))
        sess.counters.zero_()
        counts = sess.step_cfg_shared(step)
        sess.check()
        O_ref, L_ref, fresh = orc.partition_step(qc, kc, vc, sess.last_plan, S, P, cache, group=g)
        for (kk, h), items in fresh.items():       # the unconditional heads take the conditional states
            for rs, (o_f, l_f) in items:
                cache.put(kk, h + Hb, rs, o_f, l_f)
        check_out(to_np(sess.O[:Hb]), O_ref, f"cond O step {step}")
        check_lse(to_np(sess.L[:Hb]), L_ref, f"cond LSE step {step}")
        assert torch.equal(sess.O[Hb:].view(torch.int16), sess.O[:Hb].view(torch.int16))
        assert torch.equal(sess.L[Hb:], sess.L[:Hb])
        view = (lambda t: t.view(torch.int16)) if sd else (lambda t: t)
        assert torch.equal(view(sess.cache_O[:, Hb:]), view(sess.cache_O[:, :Hb]))
        assert torch.equal(sess.cache_L[:, Hb:], sess.cache_L[:, :Hb])
        c = sess.counters.cpu().numpy()
        assert int(c[0]) == counts["computed_blocks"]
        assert counts["computed_blocks"] + counts["skipped_blocks"] == \
            2 * Hb * sum(orc.n_kv_tiles(a, b) for a, b in orc.partitions(S, P)) * len(orc.query_tiles(S, P))
    # an ordinary step on both branches reuses the shared states
    qc, kc, vc = cond.next_step()
    qu, ku, vu = other.next_step()
    q, k, v = (np.concatenate([a, b]) for a, b in ((qc, qu), (kc, ku), (vc, vu)))
    sess.set_inputs(q, k, v)
    sess.step(3)
    sess.check()
    O_ref, L_ref, _ = orc.partition_step(q, k, v, sess.last_plan, S, P, cache, group=g)
    assert (sess.last_plan == orc.REUSE).any()
    check_out(to_np(sess.O), O_ref, "both branches O step 3")
    check_lse(to_np(sess.L), L_ref, "both branches LSE step 3")


def test_cfg_shared_window_mode():
    """CFG sharing in window mode: the residual made at the anchor by the
    conditional heads is the unconditional heads' residual too, so a later
    ordinary window step matches the oracle on every head."""
    Hb, S, D, W = 2, 1000, 72, 256
    cond = wl.InputStream(Hb, S, D, 0.03, seed=92)
    other = wl.InputStream(Hb, S, D, 0.5, seed=93)
    sess = Session(2 * Hb, S, D, 1, mode=dt.DT_MODE_WINDOW, window=W)
    sess.R.fill_(float("nan"))
    R = {}
    qc, kc, vc = cond.next_step()
    qu, ku, vu = other.next_step()
    sess.set_inputs(*(np.concatenate([a, b]) for a, b in ((qc, qu), (kc, ku), (vc, vu))))
    sess.step_cfg_shared(1)
    sess.check()
    O_ref, L_ref = orc.window_step(qc, kc, vc, W, True, R)
    for (h, row), val in list(R.items()):
        R[(h + Hb, row)] = val
    check_out(to_np(sess.O[:Hb]), O_ref, "cond O anchor")
    assert torch.equal(sess.R[Hb:], sess.R[:Hb])
    q, k, v = (np.concatenate([a, b]) for a, b in zip(cond.next_step(), other.next_step()))
    sess.set_inputs(q, k, v)
    sess.step(2)
    sess.check()
    O_ref, L_ref = orc.window_step(q, k, v, W, False, R)
    check_out(to_np(sess.O), O_ref, "both branches O step 2")
    check_lse(to_np(sess.L), L_ref, "both branches LSE step 2")


def test_share_previous_output():
    """Sharing across timesteps: nothing is launched; O and L keep the
    previous step's bytes and every block counts as skipped."""
    w = wl.WORKLOADS[0]
    sess = Session(w.H, w.S, w.D, w.P, reuse_per_row=2)
    s = wl.stream_for(w)
    for step in (1, 2):
        sess.set_inputs(*s.next_step())
        sess.step(step)
    sess.check()
    o, l, st = sess.O.clone(), sess.L.clone(), sess.stamps.copy()
    sess.set_inputs(*s.next_step())
    counts = sess.share_previous_output()
    sess.check()
    assert torch.equal(sess.O.view(torch.int16), o.view(torch.int16)) and torch.equal(sess.L, l)
    assert np.array_equal(sess.stamps, st)
    assert counts["computed_blocks"] == 0 and counts["computed_flops"] == 0
    assert counts["skipped_blocks"] == w.H * 8 * 8


# ------------------------------------------------- anchor-guided planning

def _sum_err(err, plan, before, anchored, S, P, g):
    """State errors of the pairs a step measured (every computed pair with a
    previous state at an anchor, else the local sets) from the kernel's
    partial sums (heads, then row groups, float64, the library's order); NaN
    where not measured.  Returns (diff, norm)."""
    nqt, nseg, H = err.shape[:3]
    diff = np.full((nqt, nseg), np.nan)
    norm = np.full((nqt, nseg), np.nan)
    tiles = orc.query_tiles(S, P)
    for t in range(nqt):
        local = 0 if g else tiles[t][0]
        for k in range(nseg):
            if plan[t, k] != orc.COMPUTE or before[t, k] < 0 or not (anchored or k == local):
                continue
            d = n = 0.0
            for h in range(H):
                for w in range(4):
                    d += float(err[t, k, h, w, 0])
                    n += float(err[t, k, h, w, 1])
            diff[t, k], norm[t, k] = d, n
    return diff, norm


@pytest.mark.parametrize("g,sd", [(0, 0), (2, 0), (0, 1)])
def test_anchor_guided_schedule_matches_oracle(g, sd):
    """DT_MODE_ANCHOR on the GPU: per step the plan and the anchor decision
    equal the oracle planner's fed with the same measurements (bit-exact);
    outputs and fresh states match the oracle run with that plan; the
    measured state errors match the oracle's own; unchanged inputs measure
    exactly zero drift; a large perturbation triggers an anchor at the next
    step and small ones do not."""
    H, S, D, P = 2, 2048, 64, 8
    sess = Session(H, S, D, P, mode=dt.DT_MODE_ANCHOR, group=g, state_dtype=sd, target_ratio=0.5,
                   drift_budget=0.5)
    nqt, nseg = sess.nqt, sess.nseg
    st_o = orc.AnchorState(nqt, nseg, 0.5, 0.5)
    stamps_o = np.full((nqt, nseg), -1, np.int32)
    cache = orc.StateCache(bf16=sd == dt.DT_STATE_BF16)
    rng = np.random.Generator(np.random.PCG64(40 + g + sd))
    master = [rng.standard_normal((H, S, D)).astype(np.float32) / np.float32(8.0) for _ in range(3)]
    sigmas = [0.0, 0.0, 0.004, 0.004, 1.0, 0.004, 0.004]
    anchors, reused = [], []
    for step, sig in enumerate(sigmas, start=1):
        for m in master:
            m += np.float32(sig) * rng.standard_normal(m.shape).astype(np.float32)
        q, k, v = (wl.f32_to_bf16_bits(m) for m in master)
        sess.set_inputs(q, k, v)
        before = sess.stamps.copy()
        sess.step(step)
        plan = sess.last_plan
        plan_o, anch_o = orc.anchor_plan(st_o, stamps_o, step, S, P, g)
        np.testing.assert_array_equal(plan, plan_o)
        assert sess.last_anchored == anch_o
        anchors.append(anch_o)
        stamps_o[plan_o == orc.COMPUTE] = step
        snap = dict(cache.slots)
        O_ref, L_ref, fresh = orc.partition_step(q, k, v, plan, S, P, cache, group=g)
        check_out(to_np(sess.O), O_ref, f"O step {step}")
        check_lse(to_np(sess.L), L_ref, f"LSE step {step}")
        # measured errors against the oracle's own
        d_o, n_o = orc.state_errors(snap, fresh, S, P, nseg)
        d_g, n_g = _sum_err(sess.last_err, plan, before, anch_o, S, P, g)
        tracked = ~np.isnan(d_g)
        assert tracked.any() or step == 1
        e_g = np.sqrt(d_g[tracked] / n_g[tracked])
        e_o = np.sqrt(d_o[tracked] / n_o[tracked])
        np.testing.assert_allclose(e_g, e_o, rtol=0.05, atol=3e-3)
        if sig == 0.0 and step > 1 and sd == dt.DT_STATE_F32:
            assert np.all(d_g[tracked] == 0.0)          # identical inputs: the kernel reproduces its states exactly
        # the oracle planner follows the same measurements
        orc.anchor_update(st_o, step, anch_o, before, d_g, n_g, S, P, g,
                          w_now=sess.weights if anch_o else None)
        np.testing.assert_array_equal(sess.anchor_arrays["alpha"][:nqt], st_o.alpha)
        np.testing.assert_array_equal(sess.anchor_arrays["drift"][:nqt], st_o.drift)
        reused.append(int((plan == orc.REUSE).sum()))
    assert anchors[0] and anchors[5] and not any(anchors[1:5])
    assert reused[1] > 0 and reused[6] > 0              # steps after an anchor reuse states
