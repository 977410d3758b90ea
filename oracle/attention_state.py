"""Plain float64 oracle of the attention-state reuse step (test infrastructure).

TEST INFRASTRUCTURE ONLY -- see the package docstring.  Slow and obviously
correct: numpy float64, a library matmul as the only "primitive", no blocking
beyond the 128-row query/key tiles that the plan itself is defined on.

Sources (cited by page title and the part of the page):
  [DT]  "DiTango: Cost-Effective Parallel Diffusion Generation with Selective
        Attention State Reuse" -- the attention-state definition (Eq. 1-3),
        composability of states (Eq. 4), the selective compute/reuse mechanism
        (Fig. 6 example, CP=4, rank 0), grouping and anchor steps (Eq. 8-9,
        Algorithm 1).  The display equations were lost from the page text;
        the readings below are the plainest ones the surrounding prose allows.
  [DFA] "DiTFastAttn: Attention Compression for Diffusion Transformer Models"
        (summary page, "Approach"): window attention plus a cached
        full-minus-window residual.

Readings taken where the pages are silent (each also listed in the design
notes of the repository):
  * state = (OUT, LSE) with OUT normalised by the partition's own softmax
    denominator and LSE the natural-log log-sum-exp of the scaled logits;
  * softmax scale 1/sqrt(D) on q.k;
  * partitions are contiguous: c = ceil(S/P), partition k = [k c, min((k+1)c, S));
  * query tiles are 128-row, partition-local; every row of a tile shares the
    tile's plan row;
  * proximity plan: for query partition q the r partitions farthest from q
    are reused, ties broken towards the lower index; q itself is always
    computed; step 1 is an anchor (everything computed);
  * window: key j is in the window of query i iff |i - j| <= W // 2 on the
    flattened token order, no wrap-around;
  * state grouping with group size g: groups of g adjacent partitions,
    G_i = [i g, min((i+1) g, P)); a query in partition q has the key sets
    {q} (its local state, handled separately) and G_i without q for every i
    (the group holding q keeps g - 1 partitions); one composed state is
    cached per (query tile, key set) and the plan decides per key set; the
    proximity plan reuses the r groups farthest from q's group (lower index
    first among equal distances) and always computes {q};
  * a bf16 state cache stores OUT rounded to nearest-even bf16 and LSE in
    float64 (fp32 on the GPU);
  * partition importance w(k) of a key set for a query tile is the normalised
    composition weight exp(LSE_k - LSE) (the share of a row's softmax mass in
    that set), averaged over the tile's rows and the heads, measured when all
    sets are fresh (an anchor step); the predicted error of reusing set k is
    ASE = w(k) * tau with tau = t - t_c its cache age (error growing linearly
    with age at a common rate); the importance plan reuses the r sets of
    smallest ASE, never the local set nor a never-written slot, lower index
    first among equal values, the products taken in float32 as the GPU-side
    weights are float32;
  * anchor-guided planning (the selection strategy's anchor condition, scale
    ratios and adapted threshold; equations lost): the state error of a key
    set k computed at step t is the relative difference ||OUT_t - OUT_c|| /
    ||OUT_t|| (Frobenius, over the tile's rows and all heads) between the
    fresh OUT and the OUT its cache slot held; the local drift of a tile is
    the state error of its own set (computed every step); an anchor is
    taken at step 1 and when the local drift accumulated since the last
    anchor exceeds a budget theta for any tile (replacing a static maximum
    age); at an anchor the scale ratio of every other set with a previous
    state is its state error per step of cache age, alpha = e / (t - t_c)
    (linear growth with age), and the threshold epsilon is the rho-quantile
    of the global importance-weighted rates w * alpha over all (tile, set)
    pairs (rho the target reuse ratio); between anchors a set is reused iff
    w * alpha * (t - t_c) <= epsilon (float32 products), never the local set
    nor a never-written slot; before the first measured anchor alpha = 1;
  * Dynamic Group State Compose by a factor k: the new group i is old groups
    k i .. k i + k - 1, its cached state their composition, its stamp the
    oldest of theirs (never written if any was never written).
"""

from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

TILE = 128
REUSE = 0
COMPUTE = 1

MODE_ALL_COMPUTE = 0
MODE_PROXIMITY = 1
MODE_ALL_REUSE = 2
MODE_EXPLICIT = 3
MODE_WINDOW = 4
MODE_IMPORTANCE = 5
MODE_ANCHOR = 6

__all__ = [
    "TILE", "REUSE", "COMPUTE", "MODE_ALL_COMPUTE", "MODE_PROXIMITY",
    "MODE_ALL_REUSE", "MODE_EXPLICIT", "MODE_WINDOW", "CacheEmpty",
    "widen_bf16", "round_bf16", "partitions", "query_tiles", "n_kv_tiles",
    "attention_state", "identity_state", "compose", "compose_n",
    "proximity_row", "build_plan", "window_in", "StateCache",
    "partition_step", "window_step", "softmax_scale",
    "n_groups", "group_key_sets", "group_proximity_row", "key_sets_of_tile",
    "compose_groups", "MODE_IMPORTANCE", "state_importance", "importance_row",
    "MODE_ANCHOR", "state_errors", "AnchorState", "anchor_plan", "anchor_update",
]


class CacheEmpty(Exception):
    """A REUSE entry points at a cache slot that has never been written."""


# ----------------------------------------------------------------------------
# bf16 helpers (exact widening; RNE narrowing of the final output)
# ----------------------------------------------------------------------------

def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """float64 -> nearest bf16 value (ties to even), returned as float64."""
    f = np.ascontiguousarray(x, dtype=np.float64)
    # exact two-step: to float32 may double-round, so round from float64 bits.
    out = np.empty_like(f)
    flat = f.reshape(-1)
    o = out.reshape(-1)
    for i in range(0, flat.size, 1 << 20):
        blk = flat[i:i + (1 << 20)]
        m, e = np.frexp(blk)            # blk = m * 2**e, 0.5 <= |m| < 1
        q = np.ldexp(np.round(np.ldexp(m, 8)), e - 8)   # 8 significant bits
        o[i:i + (1 << 20)] = q
    return out


def softmax_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)


# ----------------------------------------------------------------------------
# Geometry  [DT] context partitioning (contiguous sequence slabs)
# ----------------------------------------------------------------------------

def partitions(S: int, P: int) -> List[Tuple[int, int]]:
    """Contiguous partitions [start, end) of the token sequence, P of them."""
    c = -(-S // P) if S > 0 else 0
    return [(min(k * c, S), min((k + 1) * c, S)) for k in range(P)]


def query_tiles(S: int, P: int, window: int = 0) -> List[Tuple[int, int, int]]:
    """Query tiles (partition index, first row, end row), 128 rows each,
    partition-local.  Window mode has one partition spanning the sequence."""
    parts = [(0, S)] if window > 0 else partitions(S, P)
    out = []
    for k, (a, b) in enumerate(parts):
        for q0 in range(a, b, TILE):
            out.append((k, q0, min(q0 + TILE, b)))
    return out


def n_kv_tiles(a: int, b: int) -> int:
    return -(-(b - a) // TILE) if b > a else 0


# ----------------------------------------------------------------------------
# [DT] attention state (Eq. 1-3) and its composition (Eq. 4)
# ----------------------------------------------------------------------------

def identity_state(n: int, D: int) -> Tuple[np.ndarray, np.ndarray]:
    """State of an empty key set: OUT = 0, LSE = -inf (the unit of compose)."""
    return np.zeros((n, D)), np.full(n, -np.inf)


def attention_state(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                    keep: Optional[np.ndarray] = None):
    """Partial attention of queries q [n,D] over keys k,v [m,D].

    s_ij = scale * q_i . k_j ;  m_i = max_j s_ij ;  l_i = sum_j exp(s_ij - m_i)
    OUT_i = sum_j exp(s_ij - m_i) v_j / l_i ;  LSE_i = m_i + ln l_i
    ``keep`` (bool [n,m]) removes pairs from the key set; a row whose key set
    is empty gets the identity state.
    """
    n, D = q.shape[0], v.shape[1] if v.ndim == 2 else q.shape[1]
    if k.shape[0] == 0:
        return identity_state(n, D)
    s = (q @ k.T) * scale
    if keep is not None:
        s = np.where(keep, s, -np.inf)
    m = s.max(axis=1)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    e = np.exp(s - m_safe[:, None])
    l = e.sum(axis=1)
    with np.errstate(invalid="ignore", divide="ignore"):
        out = (e @ v) / l[:, None]
        lse = m_safe + np.log(l)
    out[empty] = 0.0
    lse[empty] = -np.inf
    return out, lse


def compose(a, b):
    """Binary composition of two states of the same rows.

    L = M + ln(e^(L1-M) + e^(L2-M)),  M = max(L1, L2)
    OUT = e^(L1-L) OUT1 + e^(L2-L) OUT2;  (0, -inf) when both are empty.
    """
    (o1, l1), (o2, l2) = a, b
    M = np.maximum(l1, l2)
    both_empty = ~np.isfinite(M)
    Ms = np.where(both_empty, 0.0, M)
    w1 = np.exp(l1 - Ms)
    w2 = np.exp(l2 - Ms)
    with np.errstate(divide="ignore"):
        L = Ms + np.log(w1 + w2)
    L = np.where(both_empty, -np.inf, L)
    Ls = np.where(both_empty, 0.0, L)
    c1 = np.where(both_empty, 0.0, np.exp(l1 - Ls))
    c2 = np.where(both_empty, 0.0, np.exp(l2 - Ls))
    return c1[:, None] * o1 + c2[:, None] * o2, L


def compose_n(states: Sequence[Tuple[np.ndarray, np.ndarray]]):
    """N-way composition: one max over all N LSEs, then one weighted pass."""
    L = np.stack([s[1] for s in states])            # [N, n]
    M = L.max(axis=0)
    empty = ~np.isfinite(M)
    Ms = np.where(empty, 0.0, M)
    w = np.exp(L - Ms[None, :])                      # [N, n]
    tot = w.sum(axis=0)
    with np.errstate(divide="ignore", invalid="ignore"):
        Lout = np.where(empty, -np.inf, Ms + np.log(tot))
        c = np.where(empty[None, :], 0.0, w / tot[None, :])
    out = np.zeros_like(states[0][0])
    for i, s in enumerate(states):
        out += c[i][:, None] * s[0]
    return out, Lout


# ----------------------------------------------------------------------------
# Plans  [DT] selective compute/reuse (Fig. 6), spatial proximity (Fig. 5a),
#        anchor steps; [DFA] window + residual as a two-key-set plan
# ----------------------------------------------------------------------------

def proximity_row(q: int, P: int, r: int) -> np.ndarray:
    """Plan row of query partition q: the r farthest partitions are reused
    (lower index first among equal distances); q itself is always computed."""
    row = np.full(P, COMPUTE, dtype=np.uint8)
    others = sorted((k for k in range(P) if k != q), key=lambda k: (-abs(q - k), k))
    for k in others[:r]:
        row[k] = REUSE
    return row


def window_in(i: np.ndarray, j: np.ndarray, W: int) -> np.ndarray:
    """[DFA] key j lies in the window of query i iff |i - j| <= W // 2."""
    return np.abs(i[:, None] - j[None, :]) <= (W // 2)


def _window_tile_blocks(q0: int, q1: int, S: int, W: int):
    """(band blocks, total blocks) of one query tile: a 128x128 block is in the
    band iff at least one of its (query, key) pairs lies in the window."""
    hw = W // 2
    nkt = n_kv_tiles(0, S)
    band = 0
    for t in range(nkt):
        a, b = t * TILE, min(t * TILE + TILE, S) - 1
        if a - (q1 - 1) <= hw and q0 - b <= hw:
            band += 1
    return band, nkt


def _window_pairs(q0: int, q1: int, S: int, W: int) -> int:
    hw = W // 2
    tot = 0
    for i in range(q0, q1):
        tot += min(S - 1, i + hw) - max(0, i - hw) + 1
    return tot


def n_groups(P: int, g: int) -> int:
    """[DT] grouping: m = ceil(P / g) groups of g adjacent partitions."""
    return -(-P // g)


def group_key_sets(q: int, P: int, g: int) -> List[List[int]]:
    """[DT] grouping: key sets of a query in partition q, as lists of
    partitions.  Set 0 is the local partition {q}; set 1 + i is group
    G_i = partitions [i g, min((i+1) g, P)) without q, so the group that
    holds q has g - 1 partitions (none when g = 1)."""
    sets = [[q]]
    for i in range(n_groups(P, g)):
        sets.append([k for k in range(i * g, min((i + 1) * g, P)) if k != q])
    return sets


def group_proximity_row(q: int, P: int, g: int, r: int) -> np.ndarray:
    """Plan row over the 1 + m key sets of a query in partition q: the local
    set is always computed; the r groups farthest from q's group q // g are
    reused, lower index first among equal distances."""
    m = n_groups(P, g)
    row = np.full(1 + m, COMPUTE, dtype=np.uint8)
    lg = q // g
    for i in sorted(range(m), key=lambda i: (-abs(i - lg), i))[:r]:
        row[1 + i] = REUSE
    return row


def key_sets_of_tile(q: int, P: int, group: int) -> List[List[int]]:
    """Key sets (lists of partitions) of a query tile in partition q: one per
    partition without grouping (group = 0), else the grouped sets."""
    return [[k] for k in range(P)] if group == 0 else group_key_sets(q, P, group)


def importance_row(w_row: np.ndarray, stamps_row: np.ndarray, step: int, r: int, local: int) -> np.ndarray:
    """[DT] error model and selection: predicted error of reusing key set k
    is w(k) * (step - t_c(k)); the r sets with the smallest predicted error
    are reused (lower index first among equal values).  The local set and
    slots never written (t_c < 0) are always computed."""
    n = len(w_row)
    row = np.full(n, COMPUTE, dtype=np.uint8)
    cand = []
    for k in range(n):
        if k == local or stamps_row[k] < 0:
            continue
        ase = np.float32(w_row[k]) * np.float32(step - int(stamps_row[k]))
        cand.append((float(ase), k))
    for _, k in sorted(cand)[:r]:
        row[k] = REUSE
    return row


def build_plan(mode: int, H: int, S: int, D: int, P: int, step: int,
               r: int = 0, window: int = 0,
               stamps: Optional[np.ndarray] = None,
               explicit: Optional[np.ndarray] = None, group: int = 0,
               weights: Optional[np.ndarray] = None):
    """Plan, block counts, algorithmic FLOPs and updated stamps of one step.

    Returns ``(plan uint8 [nqt][nseg], counts, stamps')`` where nseg = P (2 in
    window mode: key sets "window" and "complement"; 1 + ceil(P / group) with
    grouping, where r counts groups), counts =
    {computed_blocks, skipped_blocks, computed_flops}.  Step 1 of the proximity
    and window modes is an anchor: everything is computed.  A REUSE entry whose
    stamp is -1 raises ``CacheEmpty``; COMPUTE entries get stamp = step.
    """
    tiles = query_tiles(S, P, window)
    nqt = len(tiles)
    if mode == MODE_WINDOW:
        nseg = 2
        plan = np.full((nqt, 2), COMPUTE, dtype=np.uint8)
        if step > 1:
            plan[:, 1] = REUSE
    else:
        nseg = P if group == 0 else 1 + n_groups(P, group)
        plan = np.empty((nqt, nseg), dtype=np.uint8)
        for t, (kq, _, _) in enumerate(tiles):
            if mode == MODE_ALL_COMPUTE or (mode == MODE_PROXIMITY and step <= 1):
                plan[t] = COMPUTE
            elif mode == MODE_PROXIMITY:
                plan[t] = proximity_row(kq, P, r) if group == 0 else group_proximity_row(kq, P, group, r)
            elif mode == MODE_IMPORTANCE and step <= 1:
                plan[t] = COMPUTE
            elif mode == MODE_IMPORTANCE:
                st_row = (np.full(nseg, -1) if stamps is None else np.asarray(stamps).reshape(nqt, nseg)[t])
                plan[t] = importance_row(np.asarray(weights).reshape(nqt, nseg)[t], st_row, step, r,
                                         kq if group == 0 else 0)
            elif mode == MODE_ALL_REUSE:
                plan[t] = REUSE
            elif mode == MODE_EXPLICIT:
                plan[t] = np.asarray(explicit, dtype=np.uint8).reshape(nqt, nseg)[t]
            else:
                raise ValueError(mode)
    st = (np.full((nqt, nseg), -1, dtype=np.int32) if stamps is None
          else np.array(stamps, dtype=np.int32).reshape(nqt, nseg).copy())
    if np.any((plan == REUSE) & (st < 0)):
        raise CacheEmpty("REUSE of a cache slot that was never written")
    st[plan == COMPUTE] = step

    parts = partitions(S, P)
    cb = sb = fl = 0
    for t, (_, q0, q1) in enumerate(tiles):
        if mode == MODE_WINDOW:
            band, nkt = _window_tile_blocks(q0, q1, S, window)
            if plan[t, 1] == COMPUTE:
                cb += H * nkt
                fl += 4 * H * D * (q1 - q0) * S
            else:
                cb += H * band
                sb += H * (nkt - band)
                fl += 4 * H * D * _window_pairs(q0, q1, S, window)
        else:
            kq = tiles[t][0]
            for k, ks in enumerate(key_sets_of_tile(kq, P, group)):
                nb = H * sum(n_kv_tiles(*parts[j]) for j in ks)
                if plan[t, k] == COMPUTE:
                    cb += nb
                    fl += 4 * H * D * (q1 - q0) * sum(parts[j][1] - parts[j][0] for j in ks)
                else:
                    sb += nb
    counts = {"computed_blocks": cb, "skipped_blocks": sb, "computed_flops": fl}
    return plan, counts, st


# ----------------------------------------------------------------------------
# One denoising step of the method, for all rows or for a sample of rows
# ----------------------------------------------------------------------------

class StateCache:
    """Per-(key set, head) cached states of query rows.

    ``slots[(k, h, row)]`` = (OUT [D], LSE) for the rows tracked.  Rows are
    independent, so a sampled subset of rows can be followed through a whole
    schedule exactly.  With ``bf16`` the stored OUT is rounded to the nearest
    bf16 value (ties to even), the storage form the pages' memory argument
    assumes (a state is half the size of its partition's KV); LSE is kept
    exactly.
    """

    def __init__(self, bf16: bool = False):
        self.slots: Dict[Tuple[int, int, int], Tuple[np.ndarray, float]] = {}
        self.bf16 = bf16

    def put(self, k, h, rows, out, lse):
        out = round_bf16(out) if self.bf16 else out
        for i, r in enumerate(rows):
            self.slots[(k, h, int(r))] = (out[i].copy(), float(lse[i]))

    def get(self, k, h, rows, D):
        out = np.empty((len(rows), D))
        lse = np.empty(len(rows))
        for i, r in enumerate(rows):
            o, l = self.slots[(k, h, int(r))]
            out[i], lse[i] = o, l
        return out, lse


def _tile_of_rows(tiles, rows):
    starts = np.array([t[1] for t in tiles])
    return np.searchsorted(starts, rows, side="right") - 1


def partition_step(Q: np.ndarray, K: np.ndarray, V: np.ndarray, plan: np.ndarray,
                   S: int, P: int, cache: StateCache,
                   heads: Optional[Sequence[int]] = None,
                   rows: Optional[np.ndarray] = None, group: int = 0):
    """[DT] One step: (O, LSE)_q = compose over k of (fresh if COMPUTE else
    cached); fresh states overwrite their slots afterwards.  Key set k is
    partition k, or with grouping (group > 0) the k-th grouped key set of the
    query's partition; the state of a set is the attention state over the
    union of its partitions' keys.

    Q, K, V: float64 [H][S][D] (or bf16 bits, widened here).  Returns
    ``(O, LSE, fresh)`` for the selected heads x rows, O in float64 (the
    caller rounds to bf16), ``fresh`` a dict (k, h) -> (rows, OUT, LSE) of the
    states computed this step.  ``cache`` is updated in place.
    """
    if Q.dtype == np.uint16:
        Q, K, V = widen_bf16(Q), widen_bf16(K), widen_bf16(V)
    H, _, D = Q.shape
    heads = list(range(H)) if heads is None else list(heads)
    rows = np.arange(S) if rows is None else np.asarray(rows)
    tiles = query_tiles(S, P)
    parts = partitions(S, P)
    tix = _tile_of_rows(tiles, rows)
    scale = softmax_scale(D)
    O = np.zeros((len(heads), len(rows), D))
    L = np.zeros((len(heads), len(rows)))
    fresh = {}
    for hi, h in enumerate(heads):
        pending = []
        for t in np.unique(tix):
            sel = np.nonzero(tix == t)[0]
            rs = rows[sel]
            states = []
            for k, ks in enumerate(key_sets_of_tile(tiles[t][0], P, group)):
                if plan[t, k] == COMPUTE:
                    keys = np.concatenate([np.arange(*parts[j]) for j in ks]).astype(np.int64) if ks else \
                        np.zeros(0, dtype=np.int64)
                    st = attention_state(Q[h, rs], K[h, keys], V[h, keys], scale)
                    pending.append((k, h, rs, st))
                    fresh.setdefault((k, h), []).append((rs, st))
                else:
                    st = cache.get(k, h, rs, D)
                states.append(st)
            o, l = states[0]
            for st in states[1:]:
                o, l = compose((o, l), st)
            O[hi, sel], L[hi, sel] = o, l
        for k, h_, rs, st in pending:
            cache.put(k, h_, rs, st[0], st[1])
    return O, L, fresh


def state_importance(cache: StateCache, L: Dict[Tuple[int, int], float], S: int, P: int, group: int,
                     heads: Sequence[int], nseg: int) -> np.ndarray:
    """[DT] partition importance w(k) per (query tile, key set): the mean over
    the tile's rows and the heads of exp(LSE_k - LSE), LSE_k the cached state
    of key set k and LSE the row's final log-sum-exp (``L[(h, row)]``).  An
    empty state or row contributes 0.  Returns float64 [nqt][nseg]."""
    tiles = query_tiles(S, P)
    w = np.zeros((len(tiles), nseg))
    for t, (_, q0, q1) in enumerate(tiles):
        for k in range(nseg):
            tot = 0.0
            for h in heads:
                for row in range(q0, q1):
                    lk = cache.slots[(k, h, row)][1]
                    lt = L[(h, row)]
                    if np.isfinite(lk) and np.isfinite(lt):
                        tot += math.exp(lk - lt)
            w[t, k] = tot / (len(heads) * (q1 - q0))
    return w


def state_errors(before: Dict[Tuple[int, int, int], Tuple[np.ndarray, float]], fresh, S: int, P: int,
                 nseg: int) -> Tuple[np.ndarray, np.ndarray]:
    """[DT] state error of the key sets computed in a step: for every
    (query tile, key set) the sums over the tile's rows, the heads and the D
    columns of (OUT_fresh - OUT_cached)^2 and of OUT_fresh^2, where
    ``before`` is the cache's slot dictionary (k, h, row) -> (OUT, LSE) taken
    before the step and ``fresh`` the dict partition_step returns.  Pairs not
    computed, or whose slot held no state, are NaN.  The relative error is
    sqrt(diff / norm).  Returns float64 [nqt][nseg] (diff, norm)."""
    tiles = query_tiles(S, P)
    starts = np.array([t[1] for t in tiles])
    diff = np.full((len(tiles), nseg), np.nan)
    norm = np.full((len(tiles), nseg), np.nan)
    for (k, h), items in fresh.items():
        for rs, (o_f, _l_f) in items:
            t = int(np.searchsorted(starts, rs[0], side="right") - 1)
            if any((k, h, int(r)) not in before for r in rs):
                continue
            o_c = np.stack([before[(k, h, int(r))][0] for r in rs])
            if np.isnan(diff[t, k]):
                diff[t, k] = norm[t, k] = 0.0
            diff[t, k] += float(np.sum((o_f - o_c) ** 2))
            norm[t, k] += float(np.sum(o_f ** 2))
    return diff, norm


class AnchorState:
    """Host state of the anchor-guided planner: importance w and scale ratio
    alpha per (query tile, key set), the local drift accumulated since the
    last anchor per query tile, the threshold epsilon, the drift budget theta
    and the target reuse ratio rho."""

    def __init__(self, nqt: int, nseg: int, rho: float, theta: float):
        self.w = np.zeros((nqt, nseg), dtype=np.float32)
        self.alpha = np.ones((nqt, nseg), dtype=np.float32)
        self.drift = np.zeros(nqt, dtype=np.float32)
        self.eps = np.float32(0.0)
        self.rho = float(np.float32(rho))      # a float32 parameter, like the library's
        self.theta = np.float32(theta)
        self.last_anchor = 0


def _local_set(S: int, P: int, group: int, t: int) -> int:
    return 0 if group else query_tiles(S, P)[t][0]


def anchor_plan(st: AnchorState, stamps: np.ndarray, step: int, S: int, P: int, group: int = 0):
    """[DT] selection strategy with anchor steps.  Returns (plan, anchored).
    An anchor (every set computed) is taken at step 1 or when any tile's
    accumulated local drift exceeds theta; otherwise set k of tile t is
    reused iff it is not the local set, its slot holds a state and
    w * alpha * (step - t_c) <= epsilon, the products in float32."""
    nqt, nseg = stamps.shape
    anchored = step <= 1 or bool(np.any(st.drift > st.theta))
    plan = np.full((nqt, nseg), COMPUTE, dtype=np.uint8)
    if anchored:
        return plan, True
    for t in range(nqt):
        loc = _local_set(S, P, group, t)
        for k in range(nseg):
            if k == loc or stamps[t, k] < 0:
                continue
            ase = np.float32(st.w[t, k]) * np.float32(st.alpha[t, k]) * np.float32(step - int(stamps[t, k]))
            if ase <= st.eps:
                plan[t, k] = REUSE
    return plan, False


def anchor_update(st: AnchorState, step: int, anchored: bool, stamps_before: np.ndarray, diff: np.ndarray,
                  norm: np.ndarray, S: int, P: int, group: int = 0, w_now: Optional[np.ndarray] = None) -> None:
    """[DT] metadata after a step: the local drift of every tile (its own
    set's state error) accumulates since the last anchor; at an anchor the
    importance is replaced by ``w_now``, every other set with a previous
    state gets alpha = e / (step - t_c), the drift restarts at zero, and
    epsilon becomes the rho-quantile of w * alpha over all (tile, non-local
    set) pairs: the ceil(rho N)-th smallest value (0 if that count is 0).
    Errors come in as (diff, norm) sums; e = sqrt(diff / norm), 0 when
    norm is 0."""
    nqt, nseg = stamps_before.shape

    def err(t, k):
        if np.isnan(diff[t, k]):
            return None
        return float(np.float32(math.sqrt(diff[t, k] / norm[t, k]))) if norm[t, k] > 0 else 0.0

    if anchored:
        st.drift[:] = 0.0
        st.last_anchor = step
        if w_now is not None:
            st.w[:] = np.asarray(w_now, dtype=np.float32)
        for t in range(nqt):
            loc = _local_set(S, P, group, t)
            for k in range(nseg):
                if k == loc or stamps_before[t, k] < 0:
                    continue
                e = err(t, k)
                if e is not None:
                    st.alpha[t, k] = np.float32(e) / np.float32(step - int(stamps_before[t, k]))
        rates = sorted(float(np.float32(st.w[t, k]) * np.float32(st.alpha[t, k]))
                       for t in range(nqt) for k in range(nseg) if k != _local_set(S, P, group, t))
        n = int(math.ceil(st.rho * len(rates) - 1e-9)) if rates else 0
        st.eps = np.float32(rates[n - 1]) if n > 0 else np.float32(0.0)
    else:
        for t in range(nqt):
            e = err(t, _local_set(S, P, group, t))
            if e is not None:
                st.drift[t] = np.float32(st.drift[t] + np.float32(e))


def _get_or_identity(cache: StateCache, k, h, rs, D):
    """A slot never written holds nothing; its stamp (-1) already marks the
    composed slot unusable, so the identity stands in for its content."""
    try:
        return cache.get(k, h, rs, D)
    except KeyError:
        return identity_state(len(rs), D)


def compose_groups(cache: StateCache, stamps: np.ndarray, P: int, g: int, kf: int,
                   heads: Sequence[int], rows: np.ndarray, S: int, D: int):
    """[DT] Dynamic Group State Compose: regroup the cached states of group
    size g into group size kf * g.  New set 0 is old set 0; new set 1 + i is
    the composition of old sets 1 + j, j = kf i .. min(kf i + kf, m) - 1.  The
    new stamp is the oldest of the merged stamps (-1 if any is -1).  Returns
    ``(new cache, new stamps)`` for the tracked heads x rows."""
    m, m2 = n_groups(P, g), n_groups(P, kf * g)
    new = StateCache()
    tiles = query_tiles(S, P)
    tix = _tile_of_rows(tiles, np.asarray(rows))
    for h in heads:
        for t in np.unique(tix):
            rs = np.asarray(rows)[tix == t]
            o, l = cache.get(0, h, rs, D)
            new.put(0, h, rs, o, l)
            for i in range(m2):
                merged = [_get_or_identity(cache, 1 + j, h, rs, D) for j in range(kf * i, min(kf * i + kf, m))]
                o, l = compose_n(merged)
                new.put(1 + i, h, rs, o, l)
    st = np.asarray(stamps).reshape(-1, 1 + m)
    st2 = np.empty((st.shape[0], 1 + m2), dtype=np.int32)
    st2[:, 0] = st[:, 0]
    for i in range(m2):
        st2[:, 1 + i] = st[:, 1 + kf * i: 1 + min(kf * i + kf, m)].min(axis=1)
    return new, st2


def window_step(Q: np.ndarray, K: np.ndarray, V: np.ndarray, W: int,
                make_residual: bool, R: Optional[Dict[Tuple[int, int], np.ndarray]],
                heads: Optional[Sequence[int]] = None,
                rows: Optional[np.ndarray] = None):
    """[DFA] window attention with a cached residual.

    make_residual (anchor step): full = window (+) complement,
    R = OUT_full - OUT_window, O = OUT_full, LSE = LSE_full.
    otherwise: O = OUT_window + R, LSE = LSE_window.
    R is a dict (h, row) -> [D] float64, updated in place when made.
    """
    if Q.dtype == np.uint16:
        Q, K, V = widen_bf16(Q), widen_bf16(K), widen_bf16(V)
    H, S, D = Q.shape
    heads = list(range(H)) if heads is None else list(heads)
    rows = np.arange(S) if rows is None else np.asarray(rows)
    scale = softmax_scale(D)
    keys = np.arange(S)
    O = np.zeros((len(heads), len(rows), D))
    L = np.zeros((len(heads), len(rows)))
    for hi, h in enumerate(heads):
        for i0 in range(0, len(rows), TILE):
            rs = rows[i0:i0 + TILE]
            inside = window_in(rs, keys, W)
            win = attention_state(Q[h, rs], K[h], V[h], scale, keep=inside)
            if make_residual:
                comp = attention_state(Q[h, rs], K[h], V[h], scale, keep=~inside)
                full = compose(win, comp)
                res = full[0] - win[0]
                for j, r in enumerate(rs):
                    R[(h, int(r))] = res[j].copy()
                O[hi, i0:i0 + len(rs)], L[hi, i0:i0 + len(rs)] = full
            else:
                res = np.stack([R[(h, int(r))] for r in rs])
                O[hi, i0:i0 + len(rs)] = win[0] + res
                L[hi, i0:i0 + len(rs)] = win[1]
    return O, L
