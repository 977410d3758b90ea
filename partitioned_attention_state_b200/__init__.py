"""Partitioned attention-state reuse on B200 (sm_100a): Python binding of libdt.

This module only marshals arguments to the C ABI declared in ``include/dt.h``
(same function names).  Every step of the path runs in libdt: the host plan
builder and the CUDA kernels.  There is no fallback: if the library is
missing, every call raises.

Tensors are torch tensors for device memory (``torch.cuda`` streams are passed
through as raw ``cudaStream_t``); plans and stamps are numpy arrays (host).
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

__all__ = [
    "DtError", "PlanParams", "Plan", "lib_path", "load", "dt_status_string",
    "dt_plan_geometry", "dt_plan_build", "dt_attn_partial_fused", "dt_attn_partial_fused_heads", "dt_state_merge",
    "dt_state_cache_update", "dt_group_compose", "dt_window_residual", "dt_set_wait_limit_ns",
    "DT_OK", "DT_ERR_INVALID", "DT_ERR_UNSUPPORTED", "DT_ERR_CACHE_EMPTY", "DT_ERR_CUDA",
    "DT_ERR_TIMEOUT", "DT_MODE_ALL_COMPUTE", "DT_MODE_PROXIMITY", "DT_MODE_ALL_REUSE",
    "DT_MODE_EXPLICIT", "DT_MODE_WINDOW", "DT_PLAN_REUSE", "DT_PLAN_COMPUTE", "DT_WR_MAKE",
    "DT_WR_APPLY", "DT_TILE", "DT_STATE_F32", "DT_STATE_BF16", "DT_MODE_IMPORTANCE",
    "dt_plan_build_importance", "dt_state_importance", "dt_share_output", "dt_key_set_tiles",
    "dt_attn_cfg_shared", "dt_plan_share_counts", "DT_SHARE_CFG", "DT_SHARE_TIMESTEP",
    "DT_MODE_ANCHOR", "AnchorState", "dt_anchor_init", "dt_plan_build_anchor", "dt_anchor_update",
    "dt_attn_partial_fused_tracked",
]

DT_OK, DT_ERR_INVALID, DT_ERR_UNSUPPORTED, DT_ERR_CACHE_EMPTY, DT_ERR_CUDA, DT_ERR_TIMEOUT = 0, -1, -2, -3, -4, -5
DT_MODE_IMPORTANCE = 5
DT_MODE_ANCHOR = 6
DT_STATE_F32, DT_STATE_BF16 = 0, 1
DT_MODE_ALL_COMPUTE, DT_MODE_PROXIMITY, DT_MODE_ALL_REUSE, DT_MODE_EXPLICIT, DT_MODE_WINDOW = 0, 1, 2, 3, 4
DT_PLAN_REUSE, DT_PLAN_COMPUTE = 0, 1
DT_WR_MAKE, DT_WR_APPLY = 0, 1
DT_SHARE_CFG, DT_SHARE_TIMESTEP = 0, 1
DT_TILE = 128


class DtError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {dt_status_string(status)} ({status})")


class PlanParams(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("S", ctypes.c_int32), ("D", ctypes.c_int32), ("P", ctypes.c_int32),
                ("mode", ctypes.c_int32), ("reuse_per_row", ctypes.c_int32), ("window", ctypes.c_int32),
                ("step", ctypes.c_int32), ("group", ctypes.c_int32), ("state_dtype", ctypes.c_int32)]


class Plan(ctypes.Structure):
    _fields_ = [("plan", ctypes.POINTER(ctypes.c_uint8)), ("stamps", ctypes.POINTER(ctypes.c_int32)),
                ("computed_blocks", ctypes.c_int64), ("skipped_blocks", ctypes.c_int64),
                ("computed_flops", ctypes.c_int64), ("nqt", ctypes.c_int32), ("nseg", ctypes.c_int32)]


class AnchorState(ctypes.Structure):
    """dt_anchor_state: the host arrays are numpy buffers kept alive by the
    Python object (see new_anchor_state)."""
    _fields_ = [("weights", ctypes.POINTER(ctypes.c_float)), ("alpha", ctypes.POINTER(ctypes.c_float)),
                ("drift", ctypes.POINTER(ctypes.c_float)), ("eps", ctypes.c_float), ("theta", ctypes.c_float),
                ("target_ratio", ctypes.c_float), ("last_anchor", ctypes.c_int32), ("anchored", ctypes.c_int32)]


_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB: Optional[ctypes.CDLL] = None


def lib_path() -> str:
    return os.path.join(_HERE, "libdt.so")


def load() -> ctypes.CDLL:
    """Load libdt.so from this package directory (raises if it is missing)."""
    global _LIB
    if _LIB is None:
        path = lib_path()
        if not os.path.exists(path):
            raise RuntimeError(f"libdt.so not built ({path}); run python -m partitioned_attention_state_b200.build")
        lib = ctypes.CDLL(path)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        pp = ctypes.POINTER(PlanParams)
        sig = {
            "dt_status_string": ([ctypes.c_int], ctypes.c_char_p),
            "dt_plan_geometry": ([pp, ctypes.POINTER(i32), ctypes.POINTER(i32)], ctypes.c_int),
            "dt_plan_build": ([pp, vp, ctypes.POINTER(Plan)], ctypes.c_int),
            "dt_attn_partial_fused": ([pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp], ctypes.c_int),
            "dt_attn_partial_fused_heads": ([pp, i32, i32] + [vp] * 12, ctypes.c_int),
            "dt_state_merge": ([i32, i32, i32, i32, vp, vp, vp, vp, vp, vp], ctypes.c_int),
            "dt_state_cache_update": ([pp, vp, vp, vp, vp, vp, vp, vp], ctypes.c_int),
            "dt_window_residual": ([i32, i32, i32, i32, vp, vp, vp, vp, vp, vp], ctypes.c_int),
            "dt_group_compose": ([pp, i32, vp, vp, vp, vp, vp], ctypes.c_int),
            "dt_plan_build_importance": ([pp, vp, ctypes.POINTER(Plan)], ctypes.c_int),
            "dt_state_importance": ([pp, vp, vp, vp, vp, vp], ctypes.c_int),
            "dt_share_output": ([i32, i32, i32, vp, vp, vp, vp, vp], ctypes.c_int),
            "dt_attn_cfg_shared": ([pp] + [vp] * 12, ctypes.c_int),
            "dt_plan_share_counts": ([pp, i32, ctypes.POINTER(Plan)], ctypes.c_int),
            "dt_anchor_init": ([pp, ctypes.POINTER(AnchorState)], ctypes.c_int),
            "dt_plan_build_anchor": ([pp, ctypes.POINTER(AnchorState), ctypes.POINTER(Plan)], ctypes.c_int),
            "dt_anchor_update": ([pp, ctypes.POINTER(AnchorState), vp, vp, vp, vp], ctypes.c_int),
            "dt_attn_partial_fused_tracked": ([pp] + [vp] * 11 + [i32, vp], ctypes.c_int),
            "dt_key_set_tiles": ([pp, i32, i32, vp, vp, i32], ctypes.c_int),
            "dt_set_wait_limit_ns": ([i64], ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            f = getattr(lib, name)
            f.argtypes, f.restype = args, res
        _LIB = lib
    return _LIB


def _check(status: int, where: str) -> None:
    if status != DT_OK:
        raise DtError(status, where)


def _ptr(t) -> Optional[int]:
    """Device/host address of a torch tensor or numpy array (None passes NULL)."""
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def dt_status_string(status: int) -> str:
    return load().dt_status_string(status).decode()


def params(H, S, D, P=1, mode=DT_MODE_ALL_COMPUTE, reuse_per_row=0, window=0, step=1, group=0,
           state_dtype=0) -> PlanParams:
    return PlanParams(H, S, D, P, mode, reuse_per_row, window, step, group, state_dtype)


def dt_plan_geometry(p: PlanParams):
    nqt, nseg = ctypes.c_int32(), ctypes.c_int32()
    _check(load().dt_plan_geometry(ctypes.byref(p), ctypes.byref(nqt), ctypes.byref(nseg)), "dt_plan_geometry")
    return nqt.value, nseg.value


def dt_plan_build(p: PlanParams, stamps: Optional[np.ndarray] = None, explicit: Optional[np.ndarray] = None):
    """Host plan of one step.  Returns (plan uint8 [nqt][nseg], counts dict);
    ``stamps`` (int32 [nqt][nseg]) is updated in place when given."""
    nqt, nseg = dt_plan_geometry(p)
    plan = np.zeros((nqt, nseg), dtype=np.uint8)
    out = Plan()
    out.plan = plan.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))
    if stamps is not None:
        assert stamps.dtype == np.int32 and stamps.flags.c_contiguous and stamps.size == nqt * nseg
        out.stamps = stamps.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    ex = None
    if explicit is not None:
        ex = np.ascontiguousarray(explicit, dtype=np.uint8)
    _check(load().dt_plan_build(ctypes.byref(p), _ptr(ex), ctypes.byref(out)), "dt_plan_build")
    return plan, {"computed_blocks": out.computed_blocks, "skipped_blocks": out.skipped_blocks,
                  "computed_flops": out.computed_flops}


def dt_plan_build_importance(p: PlanParams, weights: Optional[np.ndarray], stamps: Optional[np.ndarray] = None):
    """Importance plan of one step (p.mode = DT_MODE_IMPORTANCE).  weights:
    float32 [nqt][nseg] (host).  Returns (plan, counts) like dt_plan_build;
    ``stamps`` is updated in place when given."""
    nqt, nseg = dt_plan_geometry(p)
    plan = np.zeros((nqt, nseg), dtype=np.uint8)
    out = Plan()
    out.plan = plan.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))
    if stamps is not None:
        assert stamps.dtype == np.int32 and stamps.flags.c_contiguous and stamps.size == nqt * nseg
        out.stamps = stamps.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    w = None
    if weights is not None:
        w = np.ascontiguousarray(weights, dtype=np.float32)
        assert w.size == nqt * nseg
    _check(load().dt_plan_build_importance(ctypes.byref(p), _ptr(w), ctypes.byref(out)), "dt_plan_build_importance")
    return plan, {"computed_blocks": out.computed_blocks, "skipped_blocks": out.skipped_blocks,
                  "computed_flops": out.computed_flops}


def dt_state_importance(p: PlanParams, cache_L, L, d_weights, d_status=None, stream=None) -> None:
    _check(load().dt_state_importance(ctypes.byref(p), _ptr(cache_L), _ptr(L), _ptr(d_weights), _ptr(d_status),
                                      _stream(stream)), "dt_state_importance")


def dt_key_set_tiles(p: PlanParams, qt: int, k: int):
    """Key tiles of key set k of query tile qt: list of (row0, rowend) with
    the tile's rows [row0, min(row0 + 128, rowend))."""
    n = load().dt_key_set_tiles(ctypes.byref(p), qt, k, None, None, 0)
    if n < 0:
        raise DtError(n, "dt_key_set_tiles")
    r0 = np.zeros(max(n, 1), np.int32)
    re = np.zeros(max(n, 1), np.int32)
    load().dt_key_set_tiles(ctypes.byref(p), qt, k, r0.ctypes.data, re.ctypes.data, n)
    return list(zip(r0[:n].tolist(), re[:n].tolist()))


def dt_share_output(n_heads: int, S: int, D: int, src_O, src_L, dst_O, dst_L, stream=None) -> None:
    _check(load().dt_share_output(n_heads, S, D, _ptr(src_O), _ptr(src_L), _ptr(dst_O), _ptr(dst_L),
                                  _stream(stream)), "dt_share_output")


def dt_attn_cfg_shared(p: PlanParams, d_plan, Q, K, V, cache_O, cache_L, R, O, L, d_counters, d_status,
                       stream=None) -> None:
    _check(load().dt_attn_cfg_shared(ctypes.byref(p), _ptr(d_plan), _ptr(Q), _ptr(K), _ptr(V), _ptr(cache_O),
                                     _ptr(cache_L), _ptr(R), _ptr(O), _ptr(L), _ptr(d_counters), _ptr(d_status),
                                     _stream(stream)), "dt_attn_cfg_shared")


def dt_plan_share_counts(p: PlanParams, kind: int, counts: Optional[dict] = None) -> dict:
    """Counts of a step under attention sharing (DT_SHARE_CFG: from the
    counts of the step's plan over all heads; DT_SHARE_TIMESTEP: nothing
    computed)."""
    io = Plan()
    if counts is not None:
        io.computed_blocks = counts["computed_blocks"]
        io.skipped_blocks = counts["skipped_blocks"]
        io.computed_flops = counts["computed_flops"]
    _check(load().dt_plan_share_counts(ctypes.byref(p), kind, ctypes.byref(io)), "dt_plan_share_counts")
    return {"computed_blocks": io.computed_blocks, "skipped_blocks": io.skipped_blocks,
            "computed_flops": io.computed_flops}


def new_anchor_state(p: PlanParams, target_ratio: float, theta: float):
    """A dt_anchor_state with its host arrays, initialised by dt_anchor_init.
    Returns (state, arrays) where arrays = {"weights", "alpha", "drift"} are
    the numpy views the state points into (keep them alive)."""
    nqt, nseg = dt_plan_geometry(p)
    arr = {"weights": np.zeros((max(nqt, 1), nseg), np.float32), "alpha": np.zeros((max(nqt, 1), nseg), np.float32),
           "drift": np.zeros(max(nqt, 1), np.float32)}
    fp = ctypes.POINTER(ctypes.c_float)
    st = AnchorState(arr["weights"].ctypes.data_as(fp), arr["alpha"].ctypes.data_as(fp),
                     arr["drift"].ctypes.data_as(fp), 0.0, theta, target_ratio, 0, 0)
    dt_anchor_init(p, st)
    return st, arr


def dt_anchor_init(p: PlanParams, st: AnchorState) -> None:
    _check(load().dt_anchor_init(ctypes.byref(p), ctypes.byref(st)), "dt_anchor_init")


def dt_plan_build_anchor(p: PlanParams, st: AnchorState, stamps: Optional[np.ndarray] = None):
    """Anchor-guided plan of one step (p.mode = DT_MODE_ANCHOR).  Returns
    (plan, counts, anchored); ``stamps`` is updated in place when given."""
    nqt, nseg = dt_plan_geometry(p)
    plan = np.zeros((nqt, nseg), dtype=np.uint8)
    out = Plan()
    out.plan = plan.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))
    if stamps is not None:
        assert stamps.dtype == np.int32 and stamps.flags.c_contiguous and stamps.size == nqt * nseg
        out.stamps = stamps.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    _check(load().dt_plan_build_anchor(ctypes.byref(p), ctypes.byref(st), ctypes.byref(out)), "dt_plan_build_anchor")
    return plan, {"computed_blocks": out.computed_blocks, "skipped_blocks": out.skipped_blocks,
                  "computed_flops": out.computed_flops}, bool(st.anchored)


def dt_anchor_update(p: PlanParams, st: AnchorState, stamps_before: np.ndarray, plan: np.ndarray, err: np.ndarray,
                     weights_now: Optional[np.ndarray] = None) -> None:
    sb = np.ascontiguousarray(stamps_before, dtype=np.int32)
    pl = np.ascontiguousarray(plan, dtype=np.uint8)
    e = np.ascontiguousarray(err, dtype=np.float32)
    w = None if weights_now is None else np.ascontiguousarray(weights_now, dtype=np.float32)
    _check(load().dt_anchor_update(ctypes.byref(p), ctypes.byref(st), _ptr(sb), _ptr(pl), _ptr(e), _ptr(w)),
           "dt_anchor_update")


def dt_attn_partial_fused_tracked(p: PlanParams, d_plan, Q, K, V, cache_O, cache_L, O, L, d_counters, d_status,
                                  d_err, err_all: bool, stream=None) -> None:
    _check(load().dt_attn_partial_fused_tracked(ctypes.byref(p), _ptr(d_plan), _ptr(Q), _ptr(K), _ptr(V),
                                                _ptr(cache_O), _ptr(cache_L), _ptr(O), _ptr(L), _ptr(d_counters),
                                                _ptr(d_status), _ptr(d_err), 1 if err_all else 0, _stream(stream)),
           "dt_attn_partial_fused_tracked")


def dt_attn_partial_fused(p: PlanParams, d_plan, Q, K, V, cache_O, cache_L, R, O, L, d_counters, d_status,
                          stream=None) -> None:
    _check(load().dt_attn_partial_fused(ctypes.byref(p), _ptr(d_plan), _ptr(Q), _ptr(K), _ptr(V), _ptr(cache_O),
                                        _ptr(cache_L), _ptr(R), _ptr(O), _ptr(L), _ptr(d_counters),
                                        _ptr(d_status), _stream(stream)), "dt_attn_partial_fused")


def dt_attn_partial_fused_heads(p: PlanParams, head_begin: int, head_count: int, d_plan, Q, K, V, cache_O, cache_L,
                                R, O, L, d_counters, d_status, stream=None) -> None:
    _check(load().dt_attn_partial_fused_heads(ctypes.byref(p), head_begin, head_count, _ptr(d_plan), _ptr(Q), _ptr(K),
                                              _ptr(V), _ptr(cache_O), _ptr(cache_L), _ptr(R), _ptr(O), _ptr(L),
                                              _ptr(d_counters), _ptr(d_status), _stream(stream)),
           "dt_attn_partial_fused_heads")


def dt_group_compose(p: PlanParams, factor: int, stamps: Optional[np.ndarray], cache_O, cache_L, d_status=None,
                     stream=None) -> Optional[np.ndarray]:
    """Regroup the cached states of layout p (p.group = g) into group size
    g * factor in place.  ``stamps`` (int32 [nqt][1+m], host) is rewritten in
    place; the returned view is its new [nqt][1+m'] shape (None if None)."""
    if stamps is not None:
        assert stamps.dtype == np.int32 and stamps.flags.c_contiguous
    _check(load().dt_group_compose(ctypes.byref(p), factor, _ptr(stamps), _ptr(cache_O), _ptr(cache_L),
                                   _ptr(d_status), _stream(stream)), "dt_group_compose")
    if stamps is None:
        return None
    nqt = stamps.shape[0]
    m = -(-p.P // p.group)
    m2 = -(-m // factor)
    return stamps.reshape(-1)[: nqt * (1 + m2)].reshape(nqt, 1 + m2)


def dt_state_merge(N, H, S, D, O_in, L_in, O_out, L_out, d_status=None, stream=None) -> None:
    _check(load().dt_state_merge(N, H, S, D, _ptr(O_in), _ptr(L_in), _ptr(O_out), _ptr(L_out), _ptr(d_status),
                                 _stream(stream)), "dt_state_merge")


def dt_state_cache_update(p: PlanParams, d_plan, fresh_O, fresh_L, cache_O, cache_L, d_status=None,
                          stream=None) -> None:
    _check(load().dt_state_cache_update(ctypes.byref(p), _ptr(d_plan), _ptr(fresh_O), _ptr(fresh_L),
                                        _ptr(cache_O), _ptr(cache_L), _ptr(d_status), _stream(stream)),
           "dt_state_cache_update")


def dt_window_residual(op, H, S, D, O_full, O_win, R, O, d_status=None, stream=None) -> None:
    _check(load().dt_window_residual(op, H, S, D, _ptr(O_full), _ptr(O_win), _ptr(R), _ptr(O), _ptr(d_status),
                                     _stream(stream)), "dt_window_residual")


def dt_set_wait_limit_ns(ns: int) -> None:
    _check(load().dt_set_wait_limit_ns(int(ns)), "dt_set_wait_limit_ns")
