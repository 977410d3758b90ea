"""Device buffers and step sequencing around the libdt C ABI.

A ``Session`` owns the device tensors of one workload (inputs, state cache,
residual, outputs, counters, status word) and the host stamps, and runs one
denoising step as: host plan build (``dt_plan_build``) -> plan upload ->
one fused launch (``dt_attn_partial_fused``), or, from host buffers, as
head-group launches (``dt_attn_partial_fused_heads``) pipelined with their
copies.  The key sets are partitions or groups of partitions (``group``),
the cached OUT fp32 or bf16 (``state_dtype``); plans follow the proximity
rule, an explicit plan, or measured importance (``measure_importance``);
cached group states can be regrouped (``compose_groups``) and outputs shared
across CFG branches or timesteps.  torch provides the memory and the
streams; every computation happens in libdt.
"""

from __future__ import annotations

from typing import Optional

import numpy as np
import torch

from . import (DT_MODE_ANCHOR, DT_MODE_IMPORTANCE, DT_MODE_PROXIMITY, DT_MODE_WINDOW, DT_SHARE_CFG,
               DT_SHARE_TIMESTEP, dt_anchor_update, dt_attn_cfg_shared, dt_attn_partial_fused,
               dt_attn_partial_fused_heads, dt_attn_partial_fused_tracked, dt_group_compose, dt_plan_build,
               dt_plan_build_anchor, dt_plan_build_importance, dt_plan_geometry, dt_plan_share_counts,
               dt_state_importance, new_anchor_state, DtError, params)


def bf16_from_bits(bits: np.ndarray, device) -> torch.Tensor:
    """uint16 bf16 bit patterns (host) -> a bf16 tensor on `device`."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(torch.bfloat16)


class Session:
    """Buffers, host stamps and plan state of one stream of denoising steps
    of one attention layer."""

    def __init__(self, H: int, S: int, D: int, P: int = 1, mode: int = DT_MODE_PROXIMITY, reuse_per_row: int = 0,
                 window: int = 0, device: str = "cuda", cache: bool = True, group: int = 0,
                 state_dtype: int = 0, target_ratio: float = 0.5, drift_budget: float = 0.5):
        """group: 0 = one key set (and cache slot) per partition; g >= 1 =
        state grouping (the local partition, then groups of g adjacent
        partitions); reuse_per_row then counts groups.  state_dtype:
        DT_STATE_F32 or DT_STATE_BF16 (cached OUT in bf16, half the bytes).
        mode DT_MODE_ANCHOR plans every step with the anchor-guided planner
        (target_ratio: share of (tile, non-local set) pairs reused right after
        an anchor; drift_budget: accumulated local drift that triggers an
        anchor); its steps synchronise to read the measured state errors."""
        self.H, self.S, self.D, self.P = H, S, D, P
        self.mode, self.r, self.window = mode, reuse_per_row, window
        self.group = group
        self.state_dtype = state_dtype
        self.device = torch.device(device)
        win = mode == DT_MODE_WINDOW
        p = params(H, S, D, P if not win else 1, mode, reuse_per_row, window, 1, group)
        self.nqt, self.nseg = dt_plan_geometry(p)
        dev = self.device
        self.Q = torch.empty((H, S, D), dtype=torch.bfloat16, device=dev)
        self.K = torch.empty_like(self.Q)
        self.V = torch.empty_like(self.Q)
        self.O = torch.empty_like(self.Q)
        self.L = torch.empty((H, S), dtype=torch.float32, device=dev)
        if win:
            self.cache_O = self.cache_L = None
            self.R = torch.zeros((H, S, D), dtype=torch.float32, device=dev)
        else:
            ns = self.nseg
            odt = torch.bfloat16 if state_dtype == 1 else torch.float32
            self.cache_O = torch.zeros((ns, H, S, D), dtype=odt, device=dev) if cache else None
            self.cache_L = torch.full((ns, H, S), float("-inf"), dtype=torch.float32, device=dev) if cache else None
            self.R = None
        self._plan_buffers()
        self.counters = torch.zeros(4, dtype=torch.int64, device=dev)
        self.status = torch.zeros(4, dtype=torch.int32, device=dev)
        self.stamps = np.full((self.nqt, self.nseg), -1, dtype=np.int32)
        self.weights: Optional[np.ndarray] = None
        self.anchor = None
        if mode == DT_MODE_ANCHOR:
            pa = params(H, S, D, P, DT_MODE_ANCHOR, 0, 0, 1, group, state_dtype)
            self.anchor, self.anchor_arrays = new_anchor_state(pa, target_ratio, drift_budget)
            self.d_err = torch.zeros((max(self.nqt, 1), self.nseg, H, 4, 2), dtype=torch.float32, device=dev)
            self.last_err = None
            self.last_anchored = False
        self.last_counts = None
        self.last_plan = None

    def _plan_buffers(self) -> None:
        self.d_plan = torch.zeros((max(self.nqt, 1), self.nseg), dtype=torch.uint8, device=self.device)
        # two pinned host plan buffers: the plan of step t is built while the
        # upload of step t-1 may still be in flight
        self._pinned = [torch.zeros((max(self.nqt, 1), self.nseg), dtype=torch.uint8, pin_memory=True)
                        for _ in range(2)]
        self._uploaded = [None, None]
        self._turn = 0
        self._plan_read = None       # event after the last launch that read d_plan

    def compose_groups(self, factor: int = 2, shrink: bool = False) -> None:
        """Dynamic Group State Compose: regroup the cached group states into
        groups `factor` times coarser (in place on the device, stamps on the
        host); later steps plan on the coarser groups.  ``shrink`` moves the
        cache into buffers of the new size (a copy) to give memory back."""
        if self.group < 1 or self.cache_O is None or self.state_dtype != 0:
            raise ValueError("compose_groups needs a grouped session with an fp32 cache")
        p = params(self.H, self.S, self.D, self.P, self.mode, self.r, 0, 1, self.group)
        for ev in self._uploaded:
            if ev is not None:
                ev.synchronize()
        self.stamps = dt_group_compose(p, factor, self.stamps, self.cache_O, self.cache_L, self.status).copy()
        self.group *= factor
        self.nseg = self.stamps.shape[1]
        if shrink:
            self.cache_O = self.cache_O[: self.nseg].clone()
            self.cache_L = self.cache_L[: self.nseg].clone()
        self._plan_buffers()

    # -------------------------------------------------------------- inputs
    def set_inputs(self, q, k, v) -> None:
        """q, k, v: uint16 bf16 bit arrays [H][S][D] (host) or bf16 tensors."""
        for dst, src in ((self.Q, q), (self.K, k), (self.V, v)):
            if isinstance(src, np.ndarray):
                dst.copy_(bf16_from_bits(src, "cpu"))
            else:
                dst.copy_(src)

    # -------------------------------------------------------------- planning
    def plan(self, step: int, mode: Optional[int] = None, explicit: Optional[np.ndarray] = None):
        mode = self.mode if mode is None else mode
        win = mode == DT_MODE_WINDOW
        p = params(self.H, self.S, self.D, 1 if win else self.P, mode, self.r, self.window, step,
                   0 if win else self.group, 0 if win else self.state_dtype)
        if mode == DT_MODE_IMPORTANCE:
            plan, counts = dt_plan_build_importance(p, self.weights, self.stamps)
        else:
            plan, counts = dt_plan_build(p, self.stamps, explicit)
        return p, plan, counts

    def measure_importance(self) -> np.ndarray:
        """Partition importance of every (query tile, key set) from the cached
        LSEs and the last step's L (dt_state_importance).  Call it after a
        step that computed every key set (an anchor); later steps in
        DT_MODE_IMPORTANCE plan with it.  Synchronises; returns the float32
        weights [nqt][nseg] kept in ``self.weights``."""
        if self.cache_L is None or self.mode == DT_MODE_WINDOW:
            raise ValueError("importance needs a partition-mode session with a cache")
        p = params(self.H, self.S, self.D, self.P, DT_MODE_IMPORTANCE, self.r, 0, 1, self.group, self.state_dtype)
        d_w = torch.empty((max(self.nqt, 1), self.nseg), dtype=torch.float32, device=self.device)
        dt_state_importance(p, self.cache_L, self.L, d_w, self.status)
        self.weights = d_w[: self.nqt].cpu().numpy().copy()
        return self.weights

    # -------------------------------------------------------------- one step
    def step(self, step: int, mode: Optional[int] = None, explicit: Optional[np.ndarray] = None,
             stream=None) -> dict:
        """Host plan build, asynchronous plan upload, one fused launch."""
        if (self.mode if mode is None else mode) == DT_MODE_ANCHOR:
            return self._step_anchor(step, stream)
        p, plan, counts = self.plan(step, mode, explicit)
        st = torch.cuda.current_stream(self.device) if stream is None else stream
        self._upload_plan(plan, st)
        self.launch(p, st)
        self._mark_plan_read(st)
        self.last_counts, self.last_plan = counts, plan
        return counts

    def _step_anchor(self, step: int, stream=None) -> dict:
        """One anchor-guided step: dt_plan_build_anchor, the tracked fused
        launch (every computed set measured at an anchor, else the local
        sets), then the state errors and, at an anchor, the importance read
        back for dt_anchor_update.  Synchronises the stream."""
        p = params(self.H, self.S, self.D, self.P, DT_MODE_ANCHOR, 0, 0, step, self.group, self.state_dtype)
        before = self.stamps.copy()
        plan, counts, anchored = dt_plan_build_anchor(p, self.anchor, self.stamps)
        st = torch.cuda.current_stream(self.device) if stream is None else stream
        self._upload_plan(plan, st)
        dt_attn_partial_fused_tracked(p, self.d_plan, self.Q, self.K, self.V, self.cache_O, self.cache_L, self.O,
                                      self.L, self.counters, self.status, self.d_err, anchored, st)
        self._mark_plan_read(st)
        w = None
        if anchored:
            d_w = torch.empty((max(self.nqt, 1), self.nseg), dtype=torch.float32, device=self.device)
            dt_state_importance(p, self.cache_L, self.L, d_w, self.status, st)
            w = d_w[: self.nqt].cpu().numpy()
        st.synchronize()
        self.check()
        err = self.d_err[: self.nqt].cpu().numpy()
        dt_anchor_update(p, self.anchor, before, plan, err, w)
        self.last_err, self.last_anchored, self.weights = err, anchored, (w if anchored else self.weights)
        self.last_counts, self.last_plan = counts, plan
        return counts

    def _upload_plan(self, plan: np.ndarray, st) -> None:
        """Asynchronous copy of a host plan into d_plan, ordered on stream `st`
        after the previous launch that read d_plan (which may have been
        issued on another stream)."""
        if self.nqt == 0:
            return
        i = self._turn
        self._turn ^= 1
        if self._uploaded[i] is not None:
            self._uploaded[i].synchronize()      # that buffer's previous upload is done
        buf = self._pinned[i]
        buf[: self.nqt].numpy()[...] = plan
        if self._plan_read is not None:
            st.wait_event(self._plan_read)
        with torch.cuda.stream(st):
            self.d_plan[: self.nqt].copy_(buf[: self.nqt], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(st)
        self._uploaded[i] = ev

    def _mark_plan_read(self, st) -> None:
        """Record that the launches issued so far on `st` read d_plan."""
        ev = torch.cuda.Event()
        ev.record(st)
        self._plan_read = ev

    def step_host(self, step: int, q, k, v, o, lse, groups: Optional[int] = None, mode: Optional[int] = None,
                  explicit: Optional[np.ndarray] = None) -> dict:
        """One step from host inputs to host outputs.

        q, k, v: pinned host tensors [H][S][D] of bf16 (or of 16-bit integers
        holding bf16 bit patterns); o: pinned host [H][S][D] of the same kind,
        lse: pinned host float32 [H][S].  The heads are split into `groups`
        contiguous groups (default: one group per ~16 MB of inputs, at most
        16 and at most H, since each group adds a launch and five copy
        calls of fixed cost); group g is uploaded on one
        stream, computed by a head-range fused launch on a second and
        downloaded on a third, so the copies of one group overlap the
        computation of the others.  Each head is computed exactly as a whole
        step computes it.  The work is ordered after, and the current stream
        made to wait for, everything issued here: synchronise the current
        stream before reading o and lse.  Returns the plan counts."""
        dev = self.device
        cur = torch.cuda.current_stream(dev)
        if getattr(self, "_host_streams", None) is None:
            self._host_streams = tuple(torch.cuda.Stream(dev) for _ in range(3))
        up, comp, down = self._host_streams
        for st in self._host_streams:
            st.wait_stream(cur)
        p, plan, counts = self.plan(step, mode, explicit)
        self._upload_plan(plan, comp)
        H = self.H
        if groups is None:
            groups = min(16, (3 * q.numel() * q.element_size()) // (16 << 20))
        n = max(1, min(H, int(groups)))
        bounds = [H * g // n for g in range(n + 1)]

        def dev_view(d, h):
            return d if h.dtype == d.dtype else d.view(h.dtype)

        for g in range(n):
            h0, h1 = bounds[g], bounds[g + 1]
            if h1 == h0:
                continue
            with torch.cuda.stream(up):
                for d, h in ((self.Q, q), (self.K, k), (self.V, v)):
                    dev_view(d, h)[h0:h1].copy_(h[h0:h1], non_blocking=True)
                arrived = torch.cuda.Event()
                arrived.record(up)
            comp.wait_event(arrived)
            dt_attn_partial_fused_heads(p, h0, h1 - h0, self.d_plan, self.Q, self.K, self.V, self.cache_O,
                                        self.cache_L, self.R, self.O, self.L, self.counters, self.status, comp)
            done = torch.cuda.Event()
            done.record(comp)
            down.wait_event(done)
            with torch.cuda.stream(down):
                o[h0:h1].copy_(dev_view(self.O, o)[h0:h1], non_blocking=True)
                lse[h0:h1].copy_(self.L[h0:h1], non_blocking=True)
        self._mark_plan_read(comp)
        for st in self._host_streams:
            cur.wait_stream(st)
        self.last_counts, self.last_plan = counts, plan
        return counts

    def step_cfg_shared(self, step: int, mode: Optional[int] = None, explicit: Optional[np.ndarray] = None,
                        stream=None) -> dict:
        """Attention sharing across CFG branches (dt_attn_cfg_shared): the
        session's H heads are the conditional half [0, H/2) and the
        unconditional half [H/2, H) of one layer.  The conditional half is
        computed with the step's plan; its O and L, and the states it
        computed, are copied to the unconditional half (whose inputs are not
        read), so the stamps hold for every head and later steps may compute
        both halves.  Returns the counts of the whole batch, the
        unconditional half's blocks counted as skipped (dt_plan_share_counts)."""
        if self.H % 2:
            raise ValueError("CFG sharing needs an even number of heads (two branches)")
        p, plan, counts = self.plan(step, mode, explicit)
        st = torch.cuda.current_stream(self.device) if stream is None else stream
        self._upload_plan(plan, st)
        dt_attn_cfg_shared(p, self.d_plan, self.Q, self.K, self.V, self.cache_O, self.cache_L, self.R, self.O,
                           self.L, self.counters, self.status, st)
        self._mark_plan_read(st)
        out = dt_plan_share_counts(p, DT_SHARE_CFG, counts)
        self.last_counts, self.last_plan = out, plan
        return out

    def share_previous_output(self) -> dict:
        """Attention sharing across timesteps: this step takes the previous
        step's attention output, which O and L already hold.  Nothing is
        launched; plan, cache and stamps are untouched.  Returns the counts
        (every block skipped, no FLOPs; dt_plan_share_counts)."""
        win = self.mode == DT_MODE_WINDOW
        p = params(self.H, self.S, self.D, 1 if win else self.P, DT_MODE_WINDOW if win else 0, 0, self.window, 1,
                   0 if win else self.group)
        out = dt_plan_share_counts(p, DT_SHARE_TIMESTEP)
        self.last_counts = out
        return out

    def launch(self, p, stream=None) -> None:
        dt_attn_partial_fused(p, self.d_plan, self.Q, self.K, self.V, self.cache_O, self.cache_L, self.R, self.O,
                              self.L, self.counters, self.status, stream)

    def capture_step(self, step: int, mode: Optional[int] = None,
                     explicit: Optional[np.ndarray] = None) -> "StepGraph":
        """Build the plan of `step` once and capture its fused launch in a CUDA
        graph.  Replaying the graph repeats the step on the current contents of
        the session's buffers with no host work (plan build, upload, launch
        set-up), which is what small workloads are bound by.  The plan lives in
        its own device buffer, so eager steps in between do not disturb it;
        replays do not advance the host stamps."""
        p, plan, counts = self.plan(step, mode, explicit)
        gplan = torch.zeros_like(self.d_plan)
        if self.nqt > 0:
            gplan[: self.nqt].copy_(torch.from_numpy(np.ascontiguousarray(plan)))
        # one eager launch first: per-process set-up (kernel attributes) stays out of the capture
        dt_attn_partial_fused(p, gplan, self.Q, self.K, self.V, self.cache_O, self.cache_L, self.R, self.O, self.L,
                              self.counters, self.status, torch.cuda.current_stream(self.device))
        side = torch.cuda.Stream(self.device)
        side.wait_stream(torch.cuda.current_stream(self.device))
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            dt_attn_partial_fused(p, gplan, self.Q, self.K, self.V, self.cache_O, self.cache_L, self.R, self.O,
                                  self.L, self.counters, self.status, side)
        torch.cuda.current_stream(self.device).wait_stream(side)
        return StepGraph(graph, gplan, counts, plan)

    def check(self) -> None:
        """Synchronise and raise if a kernel reported a device-side error."""
        torch.cuda.synchronize(self.device)
        st = int(self.status[0].item())
        if st != 0:
            raise DtError(st, "device status")


class StepGraph:
    """A captured fused launch (see Session.capture_step)."""

    def __init__(self, graph, d_plan, counts, plan):
        self.graph, self.d_plan, self.counts, self.plan = graph, d_plan, counts, plan

    def replay(self) -> dict:
        self.graph.replay()
        return self.counts
