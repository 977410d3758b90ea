"""Device buffers and step sequencing around the libdt C ABI.

A ``Session`` owns the device tensors of one workload (inputs, state cache,
residual, outputs, counters, status word) and the host stamps, and runs one
denoising step as: host plan build (``dt_plan_build``) -> plan upload ->
one fused launch (``dt_attn_partial_fused``).  torch provides the memory and
the stream; every computation happens in libdt.
"""

from __future__ import annotations

from typing import Optional

import numpy as np
import torch

from . import (DT_MODE_PROXIMITY, DT_MODE_WINDOW, dt_attn_partial_fused, dt_plan_build, dt_plan_geometry, DtError,
               params)


def bf16_from_bits(bits: np.ndarray, device) -> torch.Tensor:
    """uint16 bf16 bit patterns (host) -> a bf16 tensor on `device`."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(torch.bfloat16)


class Session:
    def __init__(self, H: int, S: int, D: int, P: int = 1, mode: int = DT_MODE_PROXIMITY, reuse_per_row: int = 0,
                 window: int = 0, device: str = "cuda", cache: bool = True):
        self.H, self.S, self.D, self.P = H, S, D, P
        self.mode, self.r, self.window = mode, reuse_per_row, window
        self.device = torch.device(device)
        win = mode == DT_MODE_WINDOW
        p = params(H, S, D, P if not win else 1, mode, reuse_per_row, window, 1)
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
            self.cache_O = torch.zeros((P, H, S, D), dtype=torch.float32, device=dev) if cache else None
            self.cache_L = torch.full((P, H, S), float("-inf"), dtype=torch.float32, device=dev) if cache else None
            self.R = None
        self.d_plan = torch.zeros((max(self.nqt, 1), self.nseg), dtype=torch.uint8, device=dev)
        # two pinned host plan buffers: the plan of step t is built while the
        # upload of step t-1 may still be in flight
        self._pinned = [torch.zeros((max(self.nqt, 1), self.nseg), dtype=torch.uint8, pin_memory=True)
                        for _ in range(2)]
        self._uploaded = [None, None]
        self._turn = 0
        self.counters = torch.zeros(4, dtype=torch.int64, device=dev)
        self.status = torch.zeros(4, dtype=torch.int32, device=dev)
        self.stamps = np.full((self.nqt, self.nseg), -1, dtype=np.int32)
        self.last_counts = None
        self.last_plan = None

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
        p = params(self.H, self.S, self.D, 1 if win else self.P, mode, self.r, self.window, step)
        plan, counts = dt_plan_build(p, self.stamps, explicit)
        return p, plan, counts

    # -------------------------------------------------------------- one step
    def step(self, step: int, mode: Optional[int] = None, explicit: Optional[np.ndarray] = None,
             stream=None) -> dict:
        """Host plan build, asynchronous plan upload, one fused launch."""
        p, plan, counts = self.plan(step, mode, explicit)
        if self.nqt > 0:
            i = self._turn
            self._turn ^= 1
            if self._uploaded[i] is not None:
                self._uploaded[i].synchronize()      # that buffer's previous upload is done
            buf = self._pinned[i]
            buf[: self.nqt].numpy()[...] = plan
            st = torch.cuda.current_stream(self.device) if stream is None else stream
            with torch.cuda.stream(st):
                self.d_plan[: self.nqt].copy_(buf[: self.nqt], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(st)
            self._uploaded[i] = ev
        self.launch(p, stream)
        self.last_counts, self.last_plan = counts, plan
        return counts

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
