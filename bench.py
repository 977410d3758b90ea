"""Benchmark of the attention-state reuse step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload NAME] [--reuse R] [--no-sweep] [--no-cpu]

A step is one denoising step of the hot path: host plan build, asynchronous
plan upload and one launch of the fused kernel (partial attention of the
COMPUTE pairs, fresh-state write-back, composition with the REUSE pairs'
cached states, output).  The default workload is the 3D video DiT shape
(H=40, S=32760, D=128, P=16) at 50% reuse, run after an anchor step filled
the state cache.  Inputs (Q/K/V 1.0 GB, state cache 10.8 GB) are larger than
L2, so no L2 flush is needed between timed steps.

Multi-GPU: the path does not shard (one GPU, no collectives); N ranks run N
independent replicas and `value` is their summed throughput.

--impl reference times the CPU oracle (float64 numpy) on the host cores on a
bounded sample of the same step and reports the same metric.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "attention ms/denoise-step & TFLOP/s on computed blocks vs B200 bf16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
NOMINAL_BF16_TFLOPS = 2250.0      # B200 dense bf16, nominal (context for the measured-peak fraction)


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="video_21x30x52_h40_d128_p16")
    ap.add_argument("--reuse", type=int, default=None, help="r: partitions reused per query partition")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--host-groups", type=int, default=None,
                    help="head groups of the host-buffer step (default: the library's choice)")
    ap.add_argument("--eager", action="store_true",
                    help="launch every timed step through the host path instead of replaying a captured CUDA graph")
    ap.add_argument("--heads", type=int, default=None, help="override H (smaller profiling captures)")
    ap.add_argument("--group", type=int, default=0,
                    help="state grouping: groups of G adjacent partitions, --reuse then counts groups")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads (tiny, DiT-XL/2-like, PixArt-like, window)")
    ap.add_argument("--no-grouped", action="store_true",
                    help="skip the grouped-cache, compose, bf16-cache and importance measurements")
    return ap.parse_args()


# ----------------------------------------------------------------------------- helpers

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def max_over_ranks(values, device):
    """Element-wise max of ``values`` over all ranks of the default process
    group (the identity on one rank).  Every multi-rank time is taken this way."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_throughput(flops_per_rank, world, ms):
    """Whole-job TFLOP/s: the work of all ranks over the slowest rank's time."""
    return flops_per_rank * world / (ms * 1e-3) / 1e12


def kernel_source_hash():
    h = hashlib.sha256()
    for fn in ("attn_fused_sm100.cu", "sm100.cuh", "geometry.h", "attn_fused.h"):
        with open(os.path.join(ROOT, "partitioned_attention_state_b200", "csrc", fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, r, group=0):
    """DRAM bytes per launch of the fused kernel from a committed ncu summary,
    valid only while the kernel sources are unchanged since the capture."""
    suffix = f"_g{group}" if group else ""
    path = os.path.join(ROOT, "profiles", f"attn_fused_sm100_{workload}{suffix}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_hash = re.search(r"kernel_source_sha256:\s*([0-9a-f]+)", text)
    m_b = re.search(rf"dram_bytes_per_launch_r{r}:\s*([0-9.eE+]+)", text)
    if not m_hash or not m_b or m_hash.group(1) != kernel_source_hash():
        return None
    return float(m_b.group(1))


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.out = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is None:
            return
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            self.out = ""

    def summary(self):
        if not self.out:
            return None
        sms, maxes, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sms.append(float(parts[1]))
                maxes.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sms:
            return None
        busy = [s for s in sms if s > 0.5 * max(sms)]
        return {"sm_mhz": float(np.median(busy)), "sm_max_mhz": max(maxes), "reasons": sorted(reasons),
                "samples": len(sms)}


# ----------------------------------------------------------------------------- oracle leg

def oracle_sample(w, r, budget_s=12.0, heads=(0,), inputs=None, group=0):
    """Time the CPU oracle on a bounded sample of one reuse step: whole query
    tiles (all their computed partial states, cached-state merges and the
    cache update) of one head, until about budget_s seconds of work."""
    import oracle as orc
    from partitioned_attention_state_b200 import workloads as wl
    try:
        from threadpoolctl import threadpool_info
        threads = max([d.get("num_threads", 1) for d in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    if inputs is None:
        s = wl.InputStream(w.H, w.S, w.D, w.sigma, seed=w.seed)
        inputs = s.next_step() + s.next_step()
    q1, k1, v1, q2, k2, v2 = inputs
    hs = list(heads)
    tiles = orc.query_tiles(w.S, w.P)
    nqt = len(tiles)
    plan1, _, st = orc.build_plan(orc.MODE_PROXIMITY, w.H, w.S, w.D, w.P, 1, r=r, group=group)
    plan2, counts, _ = orc.build_plan(orc.MODE_PROXIMITY, w.H, w.S, w.D, w.P, 2, r=r, stamps=st, group=group)
    Q1, K1, V1 = (orc.widen_bf16(x[hs]) for x in (q1, k1, v1))
    Q2, K2, V2 = (orc.widen_bf16(x[hs]) for x in (q2, k2, v2))
    parts = orc.partitions(w.S, w.P)
    rng = np.random.Generator(np.random.PCG64(7))
    order = rng.permutation(nqt)
    flops = 0
    elapsed = 0.0
    n_tiles = 0
    for t in order:
        _, q0, qe = tiles[t]
        rows = np.arange(q0, qe)
        cache = orc.StateCache()
        orc.partition_step(Q1, K1, V1, plan1, w.S, w.P, cache, rows=rows, group=group)   # anchor (untimed)
        t0 = time.perf_counter()
        orc.partition_step(Q2, K2, V2, plan2, w.S, w.P, cache, rows=rows, group=group)
        elapsed += time.perf_counter() - t0
        sets = orc.key_sets_of_tile(tiles[t][0], w.P, group)
        flops += sum(4 * w.D * len(hs) * (qe - q0) * sum(parts[j][1] - parts[j][0] for j in ks)
                     for k, ks in enumerate(sets) if plan2[t, k])
        n_tiles += 1
        if elapsed >= budget_s:
            break
    tflops = flops / elapsed / 1e12
    step_ms = counts["computed_flops"] / (flops / elapsed) * 1e3
    ratio = counts["skipped_blocks"] / max(1, counts["skipped_blocks"] + counts["computed_blocks"])
    layout = f", groups of {group}" if group else ""
    return {"tflops": tflops, "step_ms_extrapolated": step_ms, "sample_ms": elapsed * 1e3, "threads": threads,
            "sample": f"{n_tiles} query tiles x {len(hs)} head(s) of one {int(round(100 * ratio))}%-reuse step"
                      f"{layout} ({flops / 1e9:.1f} GFLOP, {elapsed:.1f} s), float64 numpy oracle"}


def oracle_sample_window(w, budget_s=4.0, inputs=None):
    """Time the CPU oracle on a bounded sample of one window + residual step
    (steps >= 2): whole query tiles of one head, their window attention plus
    the residual add; the residual comes from an untimed anchor on the same
    rows."""
    import oracle as orc
    from partitioned_attention_state_b200 import workloads as wl
    try:
        from threadpoolctl import threadpool_info
        threads = max([d.get("num_threads", 1) for d in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    if inputs is None:
        s = wl.InputStream(w.H, w.S, w.D, w.sigma, seed=w.seed)
        inputs = s.next_step() + s.next_step()
    q1, k1, v1, q2, k2, v2 = inputs
    Q1, K1, V1 = (orc.widen_bf16(x[[0]]) for x in (q1, k1, v1))
    Q2, K2, V2 = (orc.widen_bf16(x[[0]]) for x in (q2, k2, v2))
    tiles = orc.query_tiles(w.S, 1, window=w.window)
    order = np.random.Generator(np.random.PCG64(7)).permutation(len(tiles))
    hw = w.window // 2
    flops = elapsed = 0.0
    n_tiles = 0
    for t in order:
        _, q0, qe = tiles[t]
        rows = np.arange(q0, qe)
        R = {}
        orc.window_step(Q1, K1, V1, w.window, True, R, rows=rows)          # anchor (untimed)
        t0 = time.perf_counter()
        orc.window_step(Q2, K2, V2, w.window, False, R, rows=rows)
        elapsed += time.perf_counter() - t0
        flops += 4 * w.D * sum(min(w.S - 1, i + hw) - max(0, i - hw) + 1 for i in range(q0, qe))
        n_tiles += 1
        if elapsed >= budget_s:
            break
    return {"tflops": flops / elapsed / 1e12, "threads": threads,
            "sample": f"{n_tiles} query tiles x 1 head of one window + residual step "
                      f"({flops / 1e9:.2f} GFLOP, {elapsed:.1f} s), float64 numpy oracle"}


def run_reference(args, w, r, rank, group=0):
    if rank != 0:
        return
    from partitioned_attention_state_b200 import workloads as wl
    s = wl.InputStream(w.H, w.S, w.D, w.sigma, seed=w.seed)
    inputs = s.next_step() + s.next_step()
    budget = max(2.0, min(20.0, 60.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(w, r, budget_s=budget * 0.25, inputs=inputs, group=group)
    vals, samples = [], []
    for _ in range(args.steps):
        res = oracle_sample(w, r, budget_s=budget, inputs=inputs, group=group)
        vals.append(res["tflops"])
        samples.append(res)
    v = float(np.mean(vals))
    last = samples[-1]
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
        # each timed step is a bounded sample of the workload's step: ms_per_step is
        # the sample's own time (what ran); the full step's time is extrapolated
        # from the sample's throughput and reported beside it
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": float(np.mean([s["sample_ms"] for s in samples])),
        "ms_per_full_step_extrapolated": float(np.mean([s["step_ms_extrapolated"] for s in samples])),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "H": w.H, "S": w.S, "D": w.D, "P": w.P, "group": group, "reuse_per_row": r,
                   "reuse_ratio": r / (w.P if group == 0 else -(-w.P // group))},
        "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": last["threads"], "kind": "oracle",
                         "sample": last["sample"]},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- native leg

def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    from partitioned_attention_state_b200 import workloads as wl
    w = wl.BY_NAME[args.workload]
    if args.heads is not None:
        import dataclasses
        w = dataclasses.replace(w, H=args.heads, name=f"{w.name}_h{args.heads}")
    grp = args.group if w.mode == "proximity" else 0
    n_sets = w.P if grp == 0 else -(-w.P // grp)        # reusable key sets per query tile
    r = args.reuse if args.reuse is not None else (n_sets // 2 if w.mode == "proximity" else 0)

    if args.impl == "reference":
        if world > 1 and rank != 0:
            return
        run_reference(args, w, r, rank, grp)
        return

    import torch
    import torch.distributed as dist
    import partitioned_attention_state_b200 as dt
    from partitioned_attention_state_b200.session import Session

    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dt.load()
    assert args.warmup >= 3, "at least 3 warm-up steps"

    win = w.mode == "window"
    sess = Session(w.H, w.S, w.D, w.P, mode=dt.DT_MODE_WINDOW if win else dt.DT_MODE_PROXIMITY, reuse_per_row=r,
                   window=w.window, group=grp)
    stream = wl.stream_for(w)
    q1, k1, v1 = stream.next_step()
    sess.set_inputs(q1, k1, v1)
    sess.step(1)                                  # anchor: fills the state cache
    sess.check()
    q2, k2, v2 = stream.next_step()
    sess.set_inputs(q2, k2, v2)
    torch.cuda.synchronize()
    cur = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def timed(n_steps, n_warm, r_use, step_no=2):
        # The repeated reuse step has a fixed plan: replay its fused launch from
        # a CUDA graph (no host work per step), unless --eager.
        sess.r = r_use
        graph = None if args.eager else sess.capture_step(step_no)
        run = graph.replay if graph is not None else (lambda: sess.step(step_no))
        for _ in range(n_warm):
            run()
        barrier()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        counts = None
        t0.record(cur)
        for i in range(n_steps):
            ev[i][0].record(cur)
            counts = run()
            ev[i][1].record(cur)
        t1.record(cur)
        barrier()
        sess.check()
        total_ms = t0.elapsed_time(t1)
        kern_ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
        total_ms, kern_ms = max_over_ranks([total_ms, kern_ms], "cuda")
        return total_ms / n_steps, kern_ms, counts

    # headline
    with ClockSampler(local) as clk:
        ms_step, kern_ms, counts = timed(args.steps, args.warmup, r)
    clocks = clk.summary()
    flops = counts["computed_flops"]
    value = job_throughput(flops, world, ms_step)
    pk, pk_kind = peaks()
    peak_tf = float(pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved = flops / (kern_ms * 1e-3) / 1e12
    traffic = recorded_traffic(w.name, r, grp)

    # reuse sweep 0/25/50/75 %
    sweep = None
    if not args.no_sweep and not win:
        sweep = {}
        for rr in sorted({0, n_sets // 4, n_sets // 2, 3 * n_sets // 4}):
            ms, km, c = timed(max(5, args.steps // 2), 3, rr)
            sweep[f"{int(round(100 * rr / n_sets))}%"] = {
                "reuse_per_row": rr, "ms_per_step": ms, "kernel_ms": km,
                "tflops": c["computed_flops"] / (km * 1e-3) / 1e12,
                "frac_of_peak": c["computed_flops"] / (km * 1e-3) / 1e12 / peak_tf,
                "frac_of_nominal": c["computed_flops"] / (km * 1e-3) / 1e12 / NOMINAL_BF16_TFLOPS,
                "ms_over_ms_r0": None,
                "computed_blocks": c["computed_blocks"], "skipped_blocks": c["skipped_blocks"]}
        # "time falls in proportion to reuse": ms(r)/ms(0) beside the computed-FLOP fraction
        base = sweep.get("0%")
        if base:
            for e in sweep.values():
                e["ms_over_ms_r0"] = e["kernel_ms"] / base["kernel_ms"]
                e["computed_fraction"] = e["computed_blocks"] / max(1, base["computed_blocks"])
        sess.r = r

    # standalone state merge over the whole cache (HBM-bound)
    merge = None
    if not win and grp == 0:
        o_out = torch.empty((w.H, w.S, w.D), dtype=torch.float32, device="cuda")
        l_out = torch.empty((w.H, w.S), dtype=torch.float32, device="cuda")
        for _ in range(3):
            dt.dt_state_merge(w.P, w.H, w.S, w.D, sess.cache_O, sess.cache_L, o_out, l_out)
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(cur)
        nm = 5
        for _ in range(nm):
            dt.dt_state_merge(w.P, w.H, w.S, w.D, sess.cache_O, sess.cache_L, o_out, l_out)
        b.record(cur)
        barrier()
        mms = a.elapsed_time(b) / nm
        nbytes = (w.P + 1) * w.H * w.S * (4 * w.D + 4)
        hbm = float(pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        merge = {"kernel": "state_merge", "ms": mms, "bytes": nbytes, "GB/s": nbytes / (mms * 1e-3) / 1e9,
                 "frac_of_hbm": nbytes / (mms * 1e-3) / 1e9 / hbm}
        del o_out, l_out

    # the same step on the grouped cache (groups of 4 partitions, half of the
    # groups reused), and the in-place regrouping of that cache 4 -> 8
    def time_session(vs):
        """Anchor, then the graph-replayed reuse step of another session over
        the same inputs: (ms per step, counts)."""
        vs.set_inputs(q1, k1, v1)
        vs.step(1)
        vs.set_inputs(q2, k2, v2)
        vs.check()
        graph = vs.capture_step(2)
        for _ in range(3):
            graph.replay()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n = max(5, args.steps // 2)
        a.record(cur)
        for _ in range(n):
            vc = graph.replay()
        b.record(cur)
        barrier()
        vs.check()
        del graph
        return max_over_ranks([a.elapsed_time(b) / n], "cuda")[0], vc

    grouped = compose = bf16c = importance = None
    if not win and grp == 0 and not args.no_grouped:
        # importance planning: weights measured at the anchor, then the step
        # reusing the r key sets of smallest importance x age
        isess = Session(w.H, w.S, w.D, w.P, reuse_per_row=r)
        isess.set_inputs(q1, k1, v1)
        isess.step(1)
        isess.check()
        pimp = dt.params(w.H, w.S, w.D, w.P, dt.DT_MODE_IMPORTANCE, r, 0, 1)
        d_w = torch.empty((isess.nqt, isess.nseg), dtype=torch.float32, device="cuda")
        for _ in range(3):
            dt.dt_state_importance(pimp, isess.cache_L, isess.L, d_w, isess.status)
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(cur)
        for _ in range(10):
            dt.dt_state_importance(pimp, isess.cache_L, isess.L, d_w, isess.status)
        b.record(cur)
        barrier()
        ims = max_over_ranks([a.elapsed_time(b) / 10], "cuda")[0]
        ibytes = (w.P + 1) * w.H * w.S * 4
        wts = isess.measure_importance()
        isess.mode = dt.DT_MODE_IMPORTANCE
        isess.set_inputs(q2, k2, v2)
        graph = isess.capture_step(2)
        for _ in range(3):
            graph.replay()
        barrier()
        a.record(cur)
        ni = max(5, args.steps // 2)
        for _ in range(ni):
            ic = graph.replay()
        b.record(cur)
        barrier()
        isess.check()
        istep = max_over_ranks([a.elapsed_time(b) / ni], "cuda")[0]
        hbm = float(pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        importance = {"kernel": "state_importance", "ms": ims, "bytes": ibytes,
                      "GB/s": ibytes / (ims * 1e-3) / 1e9, "frac_of_hbm": ibytes / (ims * 1e-3) / 1e9 / hbm,
                      "weights_row_sum_max_err": float(np.abs(wts.sum(axis=1) - 1.0).max()),
                      "plan": f"reuse the {r} key sets of smallest importance x age per query tile",
                      "ms_per_step": istep, "tflops": ic["computed_flops"] / (istep * 1e-3) / 1e12,
                      "skipped_blocks": ic["skipped_blocks"], "computed_blocks": ic["computed_blocks"],
                      "launch": "CUDA-graph replay"}
        del graph, isess, d_w
        # the same step with the cached OUT stored in bf16
        bs = Session(w.H, w.S, w.D, w.P, reuse_per_row=r, state_dtype=dt.DT_STATE_BF16)
        bms, bc = time_session(bs)
        bf16c = {"state_dtype": "bf16 OUT, fp32 LSE", "cache_bytes": w.P * w.H * w.S * (2 * w.D + 4),
                 "fp32_cache_bytes": w.P * w.H * w.S * (4 * w.D + 4), "ms_per_step": bms,
                 "tflops": bc["computed_flops"] / (bms * 1e-3) / 1e12,
                 "frac_of_peak": bc["computed_flops"] / (bms * 1e-3) / 1e12 / peak_tf,
                 "fp32_ms_per_step": ms_step, "launch": "CUDA-graph replay"}
        del bs
    if not win and grp == 0 and not args.no_grouped and w.P % 4 == 0 and w.P >= 8:
        g4, m4 = 4, w.P // 4
        gs = Session(w.H, w.S, w.D, w.P, reuse_per_row=m4 // 2, group=g4)
        gms, gc = time_session(gs)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        slot_bytes = w.H * w.S * (4 * w.D + 4)
        grouped = {"group": g4, "reuse_groups": m4 // 2, "cache_slots": 1 + m4,
                   "cache_bytes": (1 + m4) * slot_bytes, "per_partition_cache_bytes": w.P * slot_bytes,
                   "reuse_ratio": gc["skipped_blocks"] / (gc["skipped_blocks"] + gc["computed_blocks"]),
                   "ms_per_step": gms, "tflops": gc["computed_flops"] / (gms * 1e-3) / 1e12,
                   "frac_of_peak": gc["computed_flops"] / (gms * 1e-3) / 1e12 / peak_tf,
                   "per_partition_ms_per_step": ms_step, "launch": "CUDA-graph replay"}
        # regroup 4 -> 8 in place, repeatedly on the same buffers (HBM-bound)
        pc = dt.params(w.H, w.S, w.D, w.P, dt.DT_MODE_PROXIMITY, 0, 0, 1, g4)
        for _ in range(3):
            dt.dt_group_compose(pc, 2, None, gs.cache_O, gs.cache_L, gs.status)
        barrier()
        a.record(cur)
        nc = 5
        for _ in range(nc):
            dt.dt_group_compose(pc, 2, None, gs.cache_O, gs.cache_L, gs.status)
        b.record(cur)
        barrier()
        cms = max_over_ranks([a.elapsed_time(b) / nc], "cuda")[0]
        cbytes = (m4 + -(-m4 // 2)) * slot_bytes
        hbm = float(pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        compose = {"kernel": "group_compose", "from_group": g4, "to_group": 2 * g4, "ms": cms, "bytes": cbytes,
                   "GB/s": cbytes / (cms * 1e-3) / 1e9, "frac_of_hbm": cbytes / (cms * 1e-3) / 1e9 / hbm}
        del gs

    # the anchor-guided planner on this workload: a short schedule with the
    # workload's perturbation, each step planned by dt_plan_build_anchor,
    # launched with state-error tracking and followed by dt_anchor_update
    anchor_guided = None
    if not win and grp == 0 and not args.no_grouped and args.heads is None:
        asess = Session(w.H, w.S, w.D, w.P, mode=dt.DT_MODE_ANCHOR, target_ratio=0.5, drift_budget=0.25)
        astream = wl.stream_for(w)
        rows = []
        for step in range(1, 7):
            asess.set_inputs(*astream.next_step())
            a_ev, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier()
            t0 = time.perf_counter()
            a_ev.record(cur)
            c = asess.step(step)                 # synchronises: reads the measured errors back
            b_ev.record(cur)
            barrier()
            wall = (time.perf_counter() - t0) * 1e3
            rows.append({"step": step, "anchor": bool(asess.last_anchored), "ms": a_ev.elapsed_time(b_ev),
                         "wall_ms": wall, "tflops": c["computed_flops"] / (a_ev.elapsed_time(b_ev) * 1e-3) / 1e12,
                         "reuse_ratio": c["skipped_blocks"] / max(1, c["skipped_blocks"] + c["computed_blocks"]),
                         "max_drift": float(asess.anchor_arrays["drift"][: asess.nqt].max()),
                         "eps": float(asess.anchor.eps)})
        asess.check()
        non = [r for r in rows if not r["anchor"]]
        anchor_guided = {"planner": "dt_plan_build_anchor (target_ratio 0.5, drift budget 0.25)",
                         "steps": rows, "anchors": [r["step"] for r in rows if r["anchor"]],
                         "mean_ms_non_anchor": float(np.mean([r["ms"] for r in non])) if non else None,
                         "mean_reuse_ratio_non_anchor": float(np.mean([r["reuse_ratio"] for r in non])) if non else None,
                         "timing": "CUDA events around each step (tracked launch, importance at anchors, error read-back)"}
        del asess
        torch.cuda.empty_cache()

    # every other workload of the hot-path table, timed like the headline
    # (anchor step, then graph replays of the reuse step), with the CPU
    # oracle on a bounded sample of each
    configs = None
    if not args.no_configs and args.heads is None:
        configs = {}
        for ow in wl.WORKLOADS:
            if ow.name == w.name:
                continue
            owin = ow.mode == "window"
            for orr in (ow.reuse if not owin else (0,)):
                cs = Session(ow.H, ow.S, ow.D, ow.P, mode=dt.DT_MODE_WINDOW if owin else dt.DT_MODE_PROXIMITY,
                             reuse_per_row=orr, window=ow.window)
                ostream = wl.stream_for(ow)
                oq1 = ostream.next_step()
                oq2 = ostream.next_step()
                cs.set_inputs(*oq1)
                cs.step(1)
                cs.set_inputs(*oq2)
                cs.check()
                graph = cs.capture_step(2)
                for _ in range(args.warmup):
                    graph.replay()
                barrier()
                nrep = max(10, args.steps)
                evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                       for _ in range(nrep)]
                for a_, b_ in evs:
                    a_.record(cur)
                    oc = graph.replay()
                    b_.record(cur)
                barrier()
                cs.check()
                kms = max_over_ranks([float(np.median([a_.elapsed_time(b_) for a_, b_ in evs]))], "cuda")[0]
                tf = oc["computed_flops"] / (kms * 1e-3) / 1e12
                entry = {"reuse_per_row": orr, "ms_per_step": kms, "tflops": tf, "frac": tf / peak_tf,
                         "frac_of_nominal": tf / NOMINAL_BF16_TFLOPS,
                         "reuse_ratio": oc["skipped_blocks"] / max(1, oc["skipped_blocks"] + oc["computed_blocks"]),
                         "computed_flops": oc["computed_flops"], "computed_blocks": oc["computed_blocks"],
                         "skipped_blocks": oc["skipped_blocks"],
                         "timing": "median of per-launch CUDA events over graph replays"}
                del graph, cs
                torch.cuda.empty_cache()
                if rank == 0 and not args.no_cpu:
                    if owin:
                        res = oracle_sample_window(ow, budget_s=3.0, inputs=oq1 + oq2)
                    else:
                        res = oracle_sample(ow, orr, budget_s=3.0, inputs=oq1 + oq2)
                    entry["cpu_oracle"] = {"tflops": res["tflops"], "cores": res["threads"], "sample": res["sample"]}
                configs[f"{ow.name}" + (f" r={orr}" if len(ow.reuse) > 1 else "")] = entry

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        hq = [torch.from_numpy(x.view(np.int16)).pin_memory() for x in (q2, k2, v2)]
        ho = torch.empty((w.H, w.S, w.D), dtype=torch.bfloat16).pin_memory()
        hl = torch.empty((w.H, w.S), dtype=torch.float32).pin_memory()
        ke = max(3, args.steps // 2)

        def e2e_step():
            # host inputs -> host outputs through the public API: head groups
            # uploaded, computed and downloaded on three overlapping streams
            sess.step_host(2, *hq, ho, hl, groups=args.host_groups)

        for _ in range(2):
            e2e_step()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(cur)
        for _ in range(ke):
            e2e_step()
        b.record(cur)
        barrier()
        ems = max_over_ranks([a.elapsed_time(b) / ke], "cuda")[0]
        h2d = sum(x.numel() * x.element_size() for x in hq) + sess.nqt * sess.nseg
        d2h = ho.numel() * 2 + hl.numel() * 4
        e2e = {"value": job_throughput(flops, world, ems), "unit": "TFLOP/s", "ms_per_step": ems,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "pipeline": "Session.step_host: head groups uploaded, computed and downloaded on 3 streams"}

    cpu = None
    if rank == 0 and not args.no_cpu:
        res = oracle_sample(w, r, budget_s=12.0, inputs=(q1, k1, v1, q2, k2, v2), group=grp)
        cpu = {"value": res["tflops"], "unit": "TFLOP/s", "cores": res["threads"], "kind": "oracle",
               "sample": res["sample"], "ms_per_step_extrapolated": res["step_ms_extrapolated"]}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "H": w.H, "S": w.S, "D": w.D, "P": w.P, "window": w.window,
                       "group": grp, "reuse_per_row": r,
                       "reuse_ratio": counts["skipped_blocks"] / max(1, counts["skipped_blocks"] + counts["computed_blocks"]),
                       "step": "reuse step after an anchor step",
                       "launch": "eager host path" if args.eager else "CUDA-graph replay of the fused launch",
                       "computed_blocks": counts["computed_blocks"], "skipped_blocks": counts["skipped_blocks"],
                       "computed_flops": flops, "parallelism": f"replicas x{world}",
                       "l2": "inputs larger than L2 (no flush): Q/K/V and the state cache exceed 126 MB"},
            "roofline": {"bound": "tensor", "kernel": "attn_partial_fused_kernel", "achieved": achieved,
                         "peak": peak_tf, "peak_kind": f"{pk_kind} bf16 dense (burst)", "unit": "TFLOP/s",
                         "frac": achieved / peak_tf, "frac_of_nominal": achieved / NOMINAL_BF16_TFLOPS,
                         "nominal_peak": NOMINAL_BF16_TFLOPS, "traffic": traffic, "kernel_ms": kern_ms,
                         "flops_per_launch": flops,
                         # the step runs back to back under the power cap: the measured
                         # seconds-long GEMM figure, when present, as a second denominator
                         "sustained_peak": pk.get("bf16_tflops_sustained"),
                         "frac_of_sustained": (achieved / float(pk["bf16_tflops_sustained"])
                                               if pk.get("bf16_tflops_sustained") else None)},
            "gpu_launches": args.steps,
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "reuse_sweep": sweep,
            "configs": configs,
            "state_merge": merge,
            "grouped": grouped,
            "group_compose": compose,
            "bf16_state_cache": bf16c,
            "importance": importance,
            "anchor_guided": anchor_guided,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
