/*
 * dt.h -- C ABI of the partitioned attention-state library (libdt.so).
 *
 * One denoising step of a Diffusion Transformer's full attention, split over P
 * contiguous context partitions.  For every (query tile, KV partition) pair a
 * per-step plan either COMPUTEs a fresh partial attention state or REUSEs the
 * state of that pair cached at an earlier step; the output is the
 * log-sum-exp weighted composition of all P states, and fresh states
 * overwrite their cache slots.  Partitions can be grouped (one composed
 * state per group of adjacent partitions), cached states regrouped in place,
 * stored with a bf16 OUT, and plans ranked by measured partition importance
 * and cache age.  Window attention with a cached full-minus-window residual
 * is a further plan mode on the same machinery.
 *
 * Sources: "DiTango: Cost-Effective Parallel Diffusion Generation with
 * Selective Attention State Reuse" (attention state, Eq. 1-3; composition,
 * Eq. 4; selective compute and reuse, Fig. 6; anchor steps; state grouping
 * and Dynamic Group State Compose; error model and selection strategy) and
 * "DiTFastAttn: Attention Compression for Diffusion Transformer Models"
 * (summary page, Approach: window attention with residual sharing).
 *
 * Conventions for every entry point
 *   - returns an int status: DT_OK (0) or a negative DT_ERR_* code; no C++
 *     exception crosses this boundary;
 *   - the caller owns and allocates every buffer; the library allocates no
 *     device or host memory (tensor memory inside a kernel aside);
 *   - device work is enqueued asynchronously on the caller's stream
 *     (cudaStream_t passed as void*; NULL = legacy default stream);
 *   - device pointers must be 16-byte aligned; kernels report device-side
 *     errors by writing a DT_ERR_* code into *d_status (int32, device memory,
 *     caller-zeroed), which the caller reads after synchronising;
 *   - tensors are dense, row-major, batch 1:
 *       Q, K, V, O           bf16  [H][S][D]
 *       L (final LSE)        fp32  [H][S]
 *       cache_O              fp32  [nseg][H][S][D] (state OUT of key set k;
 *                                   bf16 with state_dtype = DT_STATE_BF16)
 *       cache_L              fp32  [nseg][H][S]    (state LSE of key set k)
 *       R (window residual)  fp32  [H][S][D]
 *     The state of query row s, head h, key set k (KV partition k, or the
 *     k-th grouped key set) lives at cache_O[((k*H + h)*S + s)*D + d] and
 *     cache_L[(k*H + h)*S + s]; nseg = P without grouping.
 *   - softmax scale is 1/sqrt(D); LSE is a natural logarithm; OUT is
 *     normalised by the partition's own softmax denominator.
 */
#ifndef DT_H_
#define DT_H_

#include <stdint.h>

#if defined(__GNUC__)
#define DT_API __attribute__((visibility("default")))
#else
#define DT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes -------------------------------------------------------- */
#define DT_OK               0
#define DT_ERR_INVALID     -1  /* bad argument: shape, null pointer, mode, plan value */
#define DT_ERR_UNSUPPORTED -2  /* D not in {64, 72, 128}, a misaligned pointer, more than 64
                                  key sets in the fused step, or a bf16 state cache given to a
                                  call that takes fp32 states only */
#define DT_ERR_CACHE_EMPTY -3  /* a REUSE entry names a slot never written (stamp < 0) */
#define DT_ERR_CUDA        -4  /* a CUDA runtime/driver call failed */
#define DT_ERR_TIMEOUT     -5  /* (device) a bounded wait inside a kernel ran out */

/* ---- plan modes ---------------------------------------------------------- */
#define DT_MODE_ALL_COMPUTE 0  /* every pair computed */
#define DT_MODE_PROXIMITY   1  /* step 1: anchor (all computed); later steps:
                                  the r partitions farthest from the query's own
                                  partition are reused, ties to the lower index */
#define DT_MODE_ALL_REUSE   2  /* every pair reused */
#define DT_MODE_EXPLICIT    3  /* plan copied from the caller */
#define DT_MODE_WINDOW      4  /* window + residual: 2 key sets per query tile */
#define DT_MODE_IMPORTANCE  5  /* step 1: anchor; later steps: the r key sets of smallest
                                  predicted error (importance x cache age) are reused;
                                  built by dt_plan_build_importance */
#define DT_MODE_ANCHOR      6  /* anchor-guided: anchors triggered by local drift, reuse
                                  by a threshold adapted at anchors; built by
                                  dt_plan_build_anchor (below) */

#define DT_PLAN_REUSE   0
#define DT_PLAN_COMPUTE 1

#define DT_TILE 128             /* query/key tile rows; tiles never straddle a partition */

typedef struct {
  int32_t H, S, D, P;           /* heads, tokens, head dim, partitions (P ignored in window mode) */
  int32_t mode;                 /* DT_MODE_* */
  int32_t reuse_per_row;        /* r: partitions (with grouping: groups) reused per query partition (proximity) */
  int32_t window;               /* W: key j is in query i's window iff |i-j| <= W/2 (window mode) */
  int32_t step;                 /* denoising step t, 1-based; step 1 is an anchor */
  int32_t group;                /* g: 0 = one key set per partition; g >= 1 = state grouping (below).
                                   Partition modes only (0 in window mode) */
  int32_t state_dtype;          /* element type of the cached OUT: DT_STATE_F32 or DT_STATE_BF16
                                   (partition modes; cached LSE is always fp32) */
} dt_plan_params;

#define DT_STATE_F32  0         /* cache_O is float [nseg][H][S][D] */
#define DT_STATE_BF16 1         /* cache_O is bf16 [nseg][H][S][D] (RNE from the fp32 state),
                                   half the bytes; accepted by dt_attn_partial_fused(_heads) only */

/* State grouping ("DiTango", grouping of spatially adjacent attention states;
 * the local state is handled separately): with group size g the P partitions
 * form m = ceil(P/g) groups G_i = partitions [i*g, min((i+1)*g, P)).  A query
 * tile of partition q then has nseg = 1 + m key sets: set 0 = {q}, set 1+i =
 * G_i without q (the group holding q keeps g-1 partitions, none if g = 1).
 * One state per (query tile, key set) is computed or reused and cached: a
 * group's slot holds the composition of its partitions' states.  The
 * proximity plan always computes set 0 and reuses the r groups farthest from
 * q's group q/g (|i - q/g|, equal distances lower index first; r <= m).
 * nseg must not exceed 64 for the fused kernel. */

typedef struct {
  uint8_t* plan;                /* caller-allocated host [nqt][nseg] (out) */
  int32_t* stamps;              /* caller-allocated host [nqt][nseg] (in/out): step each
                                   slot was last computed, -1 = never; NULL = all -1 */
  int64_t computed_blocks;      /* (out) 128x128 blocks whose scores are computed, x H */
  int64_t skipped_blocks;       /* (out) blocks covered by reused states, x H */
  int64_t computed_flops;       /* (out) 4*D*(query,key) pairs computed, x H */
  int32_t nqt;                  /* (out) query tiles per head */
  int32_t nseg;                 /* (out) key sets per query tile: P, 1 + ceil(P/g) with
                                   grouping, or 2 in window mode */
} dt_plan;

/* Human-readable name of a status code (static storage, never NULL). */
DT_API const char* dt_status_string(int status);

/* Number of query tiles per head and of key sets per query tile for these
 * parameters, so the caller can size dt_plan.plan / dt_plan.stamps.
 * Query tiles are 128-row, partition-local: nqt = sum_k ceil(|k|/128) with
 * partition k = [k*c, min((k+1)*c, S)), c = ceil(S/P) ("DiTango", context
 * partitioning of the sequence).  Host only.  Errors: DT_ERR_INVALID. */
DT_API int dt_plan_geometry(const dt_plan_params* p, int32_t* nqt, int32_t* nseg);

/* Key tiles of key set k of query tile qt, as the fused kernel visits them
 * (before its rotation of the visiting order): for tile i, rows
 * [row0[i], min(row0[i] + 128, rowend[i])) of K and V.  Tiles are
 * partition-local; a grouped set lists its partitions' tiles in increasing
 * partition order, skipping the query's own partition.  Window mode lists
 * the tiles of its two key sets (edge tiles then carry a band mask not
 * shown here).  Fills at most cap entries of row0 / rowend (host arrays,
 * NULL if cap = 0) and returns the number of tiles (>= 0), or DT_ERR_INVALID.
 * Host only. */
DT_API int dt_key_set_tiles(const dt_plan_params* p, int32_t qt, int32_t k, int32_t* row0, int32_t* rowend,
                     int32_t cap);

/* Build the compute/reuse plan of one step on the host ("DiTango", selective
 * compute and reuse, Fig. 6; anchor steps).  explicit_plan ([nqt][nseg],
 * values DT_PLAN_*) is read only in DT_MODE_EXPLICIT.  Window mode: key set 0
 * is the window (always computed), key set 1 its complement, computed at the
 * anchor step (which makes the residual) and reused afterwards ("DiTFastAttn",
 * window attention with residual sharing).  Validates that every REUSE entry
 * has stamp >= 0 (else DT_ERR_CACHE_EMPTY, out->plan left filled, stamps
 * untouched), then sets stamp = step on COMPUTE entries and fills the counts.
 * Host only, no CUDA call.  Errors: DT_ERR_INVALID, DT_ERR_CACHE_EMPTY. */
DT_API int dt_plan_build(const dt_plan_params* p, const uint8_t* explicit_plan, dt_plan* out);

/* Importance plan of one step ("DiTango", error model and selection
 * strategy: the error of reusing a cached state is its partition importance
 * times a growth over cache age).  p->mode must be DT_MODE_IMPORTANCE (either
 * key-set layout).  weights: host float [nqt][nseg], the importance of each
 * key set for each query tile (dt_state_importance, measured at an anchor).
 * Step 1 computes everything.  Later steps, per query tile: predicted error
 * e_k = weights[k] * (step - stamp_k), a float product; the local key set
 * (partition q, or set 0 when grouped) and slots with stamp < 0 are never
 * reused; the r = p->reuse_per_row sets of smallest e_k are reused, the lower
 * index first among equal values (fewer if fewer are eligible).  Then stamps
 * and counts as dt_plan_build.  Host only.  Errors: DT_ERR_INVALID. */
DT_API int dt_plan_build_importance(const dt_plan_params* p, const float* weights, dt_plan* out);

/* ---- anchor-guided planning ("DiTango", selection strategy and anchor
 * steps; the equations are lost, these are the readings the prose supports).
 * The state error of a key set computed at step t is ||OUT_t - OUT_c|| /
 * ||OUT_t|| (Frobenius over the query tile's rows, all heads and D), OUT_c
 * being the OUT its cache slot held; a tile's local drift is that error of
 * its own key set (partition q, or set 0 with grouping), which every step
 * computes.  An anchor (every set computed) is taken at step 1 and when the
 * drift accumulated since the last anchor exceeds theta for any tile.  At an
 * anchor the scale ratio of every other set with a previous state becomes
 * alpha = e / (t - t_c) (error per step of cache age), and epsilon becomes
 * the target_ratio-quantile of w * alpha over all (tile, non-local set)
 * pairs (the ceil(target_ratio * N)-th smallest, 0 if that count is 0).
 * Between anchors set k of a tile is reused iff it is not the local set, its
 * slot holds a state and w * alpha * (t - t_c) <= epsilon (float32 products
 * in that order). */
typedef struct {
  float* weights;             /* host [nqt][nseg]: importance w, replaced at anchors (in/out) */
  float* alpha;               /* host [nqt][nseg]: scale ratios, 1 until measured (in/out) */
  float* drift;               /* host [nqt]: local drift accumulated since the last anchor (in/out) */
  float eps;                  /* reuse threshold epsilon (in/out) */
  float theta;                /* drift budget that triggers an anchor (in) */
  float target_ratio;         /* share of (tile, non-local set) pairs reused right after an anchor (in) */
  int32_t last_anchor;        /* step of the last anchor, 0 = none (in/out) */
  int32_t anchored;           /* (out) 1 if the plan dt_plan_build_anchor built last is an anchor */
} dt_anchor_state;

/* Initial planner state: w = 0, alpha = 1, drift = 0, eps = 0, last_anchor =
 * 0, anchored = 0 (theta and target_ratio are the caller's).  The three
 * arrays are caller-allocated host memory sized by dt_plan_geometry.  Host
 * only.  Errors: DT_ERR_INVALID. */
DT_API int dt_anchor_init(const dt_plan_params* p, dt_anchor_state* a);

/* Plan of one step in DT_MODE_ANCHOR (p->mode must be DT_MODE_ANCHOR; either
 * key-set layout): an anchor or the threshold rule above; sets a->anchored;
 * then stamps and counts as dt_plan_build.  Host only.  Errors:
 * DT_ERR_INVALID. */
DT_API int dt_plan_build_anchor(const dt_plan_params* p, dt_anchor_state* a, dt_plan* out);

/* Planner metadata after a step ran through dt_attn_partial_fused_tracked
 * with the plan of dt_plan_build_anchor.  stamps_before: host [nqt][nseg],
 * the stamps before that plan was built; plan: that plan; err: host copy of
 * the step's d_err (layout below); weights_now: host [nqt][nseg] importance
 * measured after the step (dt_state_importance), used and required only
 * when a->anchored.  The error of a pair is sqrt(sum diff / sum norm) over
 * its heads and warps in increasing order (double sums), rounded to float;
 * pairs whose stamp was < 0 have no previous state and are skipped.  At an
 * anchor: drift = 0, last_anchor = step, w = weights_now, alpha and epsilon
 * as above; otherwise each tile's drift += its local error.  Host only.
 * Errors: DT_ERR_INVALID. */
DT_API int dt_anchor_update(const dt_plan_params* p, dt_anchor_state* a, const int32_t* stamps_before,
                     const uint8_t* plan, const float* err, const float* weights_now);

/* Fused step on the GPU ("DiTango", attention state Eq. 1-3, composition Eq. 4,
 * selective reuse Fig. 6).  For each head and query tile and each key set of
 * the tile's plan row (a partition, a group of partitions with p->group >= 1,
 * or a window-mode set): COMPUTE runs the partial attention (tensor cores) and
 * writes the fresh state (OUT, LSE) to its cache slot; REUSE reads the cached
 * state.  All states of the row are composed into O (bf16) and L.
 *   d_plan      device copy of dt_plan.plan, [nqt][nseg] uint8; every entry
 *               must be DT_PLAN_REUSE (0) or DT_PLAN_COMPUTE (1) (the kernel
 *               reads bit 0 of each byte; dt_plan_build writes only 0 and 1)
 *   Q, K, V     bf16 [H][S][D] (read)
 *   cache_O/L   fp32 [nseg][H][S][D] / [nseg][H][S] state slots, slot (k, h,
 *               row) for key set k (REUSE slots read, COMPUTE slots written;
 *               slots of other pairs untouched).  May be NULL in window mode.
 *   R           window mode only: fp32 [H][S][D]; written at the anchor step
 *               (R = OUT_full - OUT_window), read afterwards (O = OUT_window + R,
 *               L = LSE_window).  NULL otherwise.
 *   O, L        outputs bf16 [H][S][D], fp32 [H][S]
 *   d_counters  int64[4] device, accumulated (caller zeroes): [0] computed
 *               blocks and [1] skipped blocks (same definitions as dt_plan),
 *               [2] fresh states written and [3] cached states read, each
 *               counted per (query tile, key set, head)
 *   d_status    int32 device status word (see conventions)
 * The host validates shapes and alignment before any launch.  One launch.
 * Partition mode supports at most 64 key sets (DT_ERR_UNSUPPORTED above);
 * d_plan must be 16-byte aligned like every other pointer.  A cache_O that
 * starts on a 32-byte boundary lets the kernel store fresh fp32 states 32
 * bytes per instruction (results are identical either way). */
DT_API int dt_attn_partial_fused(const dt_plan_params* p, const uint8_t* d_plan,
                          const void* Q, const void* K, const void* V,
                          float* cache_O, float* cache_L, float* R,
                          void* O, float* L,
                          int64_t* d_counters, int32_t* d_status, void* stream);

/* The same step restricted to heads [head_begin, head_begin + head_count):
 * the arguments are those of dt_attn_partial_fused, with the buffers of all
 * p->H heads (same layouts, same pointers); only the rows of the selected
 * heads are read or written, and each is computed exactly as the whole-step
 * launch computes it (bit-identical), so launches over disjoint head ranges
 * that cover all heads equal one whole-step launch.  Lets a caller overlap
 * the host<->device copies of some heads with the computation of others.
 * The counters accumulate the selected heads only.  Errors: those of
 * dt_attn_partial_fused, and DT_ERR_INVALID for a range outside [0, H).
 * head_count = 0 launches nothing and returns DT_OK. */
DT_API int dt_attn_partial_fused_heads(const dt_plan_params* p, int32_t head_begin, int32_t head_count,
                          const uint8_t* d_plan, const void* Q, const void* K, const void* V,
                          float* cache_O, float* cache_L, float* R, void* O, float* L,
                          int64_t* d_counters, int32_t* d_status, void* stream);

/* The fused step of dt_attn_partial_fused that also measures state errors
 * for the anchor-guided planner: for every (query tile, key set) it computes
 * (all of them if err_all, else only the tile's local set) it reads the
 * slot's previous OUT before overwriting it and writes, per head and per
 * group of 32 rows (4 per tile), the sums over those rows and the D columns
 * of (OUT_new - OUT_old)^2 and OUT_new^2 to
 *   d_err fp32 [nqt][nseg][H][4][2]  (device; entries of pairs not measured
 *                                     are left as they were).
 * Partition modes only (fp32 or bf16 states).  Errors: those of
 * dt_attn_partial_fused; DT_ERR_INVALID for window mode or a null d_err. */
DT_API int dt_attn_partial_fused_tracked(const dt_plan_params* p, const uint8_t* d_plan,
                          const void* Q, const void* K, const void* V,
                          float* cache_O, float* cache_L, void* O, float* L,
                          int64_t* d_counters, int32_t* d_status,
                          float* d_err, int32_t err_all, void* stream);

/* N-way composition of states ("DiTango", composition of attention states,
 * Eq. 4): for every row, L = M + ln sum_n e^(L_n - M), M = max_n L_n,
 * OUT = sum_n e^(L_n - L) OUT_n; rows whose N inputs are all empty get
 * (0, -inf).  O_in fp32 [N][H][S][D], L_in fp32 [N][H][S] (read);
 * O_out fp32 [H][S][D], L_out fp32 [H][S] (written).  HBM-bound kernel. */
DT_API int dt_state_merge(int32_t N, int32_t H, int32_t S, int32_t D,
                   const float* O_in, const float* L_in,
                   float* O_out, float* L_out, int32_t* d_status, void* stream);

/* Plan-driven scatter of fresh states into the cache ("DiTango", freshly
 * computed states are stored in the attention state cache): for every
 * (query tile, partition k) with plan COMPUTE, copy the tile's rows of
 * fresh_O/fresh_L (layout of cache_O/cache_L) into cache_O/cache_L; REUSE
 * slots stay byte-identical.  Partition modes and fp32 states only
 * (DT_ERR_UNSUPPORTED for DT_STATE_BF16).  HBM-bound kernel. */
DT_API int dt_state_cache_update(const dt_plan_params* p, const uint8_t* d_plan,
                          const float* fresh_O, const float* fresh_L,
                          float* cache_O, float* cache_L,
                          int32_t* d_status, void* stream);

/* Dynamic Group State Compose ("DiTango", merging cached states into
 * k-times coarser groups, composability Eq. 4): regroups the cache of the
 * grouped layout p (p->group = g >= 1, partition modes) into group size
 * g*factor, in place.  New set 0 = old set 0; new set 1+i = composition of old
 * sets 1+j, j = factor*i .. min(factor*i + factor, m) - 1.  Afterwards slots
 * [0, 1 + ceil(m/factor)) of cache_O [nseg][H][S][D] / cache_L [nseg][H][S]
 * hold the coarse layout (later slots are stale), and the caller continues
 * with p->group = g*factor.  stamps (host, optional) is [nqt][1+m] on entry
 * and is rewritten as [nqt][1+m'] in its first entries: a composed slot gets
 * the oldest stamp of the slots it merges (-1 if any is -1).  One launch of an
 * HBM-bound kernel.  Errors: DT_ERR_INVALID (bad params, factor < 2 or > 8,
 * null cache), DT_ERR_UNSUPPORTED (misaligned cache pointers, bf16 states). */
DT_API int dt_group_compose(const dt_plan_params* p, int32_t factor, int32_t* stamps,
                     float* cache_O, float* cache_L, int32_t* d_status, void* stream);

/* Partition importance ("DiTango", error model: the normalised composition
 * weight of a state, Eq. 4): weights[qt][k] = mean over the query tile's rows
 * and all heads of exp(cache_L[k][h][row] - L[h][row]), the share of each
 * row's softmax mass that falls on key set k (0 where either LSE is -inf).
 * Meaningful after a step that computed every key set (an anchor), whose
 * outputs are L and whose fresh states are in cache_L.  Partition modes
 * (either layout).  cache_L fp32 [nseg][H][S], L fp32 [H][S] (read),
 * d_weights fp32 [nqt][nseg] (device, written).  One launch, HBM-bound.
 * Errors: DT_ERR_INVALID, DT_ERR_UNSUPPORTED (misaligned pointers). */
DT_API int dt_state_importance(const dt_plan_params* p, const float* cache_L, const float* L,
                        float* d_weights, int32_t* d_status, void* stream);

#define DT_WR_MAKE  0   /* R = O_full - O_win                 */
#define DT_WR_APPLY 1   /* O = bf16(O_win + R)  (O_full unused) */

/* Residual of window attention ("DiTFastAttn", window attention with
 * residual sharing): MAKE writes R (fp32 [H][S][D]) from O_full and O_win
 * (fp32 [H][S][D]); APPLY writes O (bf16 [H][S][D]) from O_win and R.
 * HBM-bound elementwise kernel. */
DT_API int dt_window_residual(int32_t op, int32_t H, int32_t S, int32_t D,
                       const float* O_full, const float* O_win,
                       float* R, void* O, int32_t* d_status, void* stream);

/* Attention sharing ("DiTFastAttn", attention sharing across CFG branches
 * and across timesteps: a branch or step takes another's attention output
 * instead of computing its own): copies the outputs of n_heads heads,
 * O bf16 [n_heads][S][D] and L fp32 [n_heads][S], from src to dst on the
 * stream (device memory; src and dst ranges must not overlap unless equal,
 * in which case nothing is done).  Errors: DT_ERR_INVALID (negative sizes,
 * null or partially overlapping buffers), DT_ERR_CUDA. */
DT_API int dt_share_output(int32_t n_heads, int32_t S, int32_t D, const void* src_O, const float* src_L,
                    void* dst_O, float* dst_L, void* stream);

/* Attention sharing across CFG branches as one step ("DiTFastAttn",
 * attention sharing across CFG: the unconditional branch takes the
 * conditional branch's attention output).  The p->H heads (H even) hold the
 * conditional branch in heads [0, H/2) and the unconditional one in
 * [H/2, H).  Runs the fused step (arguments as dt_attn_partial_fused, with
 * the plan dt_plan_build made for all H heads) on the conditional heads,
 * copies their O and L to the unconditional heads, and copies the states
 * they computed (cache slots of the COMPUTE entries; in window mode R rows
 * where the complement was computed) to the same slots of the unconditional
 * heads: the shared attention is the conditional branch's, so the stamps
 * dt_plan_build wrote stay true for every head, and a later step that
 * computes both branches reuses those states.  Unconditional inputs are not
 * read.  The counters accumulate the conditional heads' launch.  Errors:
 * those of dt_attn_partial_fused, DT_ERR_INVALID for odd H. */
DT_API int dt_attn_cfg_shared(const dt_plan_params* p, const uint8_t* d_plan,
                       const void* Q, const void* K, const void* V,
                       float* cache_O, float* cache_L, float* R, void* O, float* L,
                       int64_t* d_counters, int32_t* d_status, void* stream);

#define DT_SHARE_CFG      0   /* the conditional half computes, the unconditional half shares */
#define DT_SHARE_TIMESTEP 1   /* the step takes the previous step's output: nothing computed */

/* Counts of a step that shares attention ("DiTFastAttn", attention sharing
 * across CFG branches and across timesteps).  DT_SHARE_CFG: on entry io
 * holds the counts dt_plan_build returned for the step's plan over all p->H
 * heads (H even); on return, the counts of the step as dt_attn_cfg_shared
 * runs it (the unconditional half's blocks skipped, its FLOPs not spent).
 * DT_SHARE_TIMESTEP: io's counts become zero computed blocks and FLOPs and
 * every block of every head skipped (counts on entry ignored).  io->plan and
 * io->stamps are neither read nor written.  Host only.  Errors:
 * DT_ERR_INVALID (bad params, unknown kind, odd H for DT_SHARE_CFG). */
DT_API int dt_plan_share_counts(const dt_plan_params* p, int32_t kind, dt_plan* io);

/* Limit, in nanoseconds, of every bounded wait inside the fused kernel
 * (default 2e9).  A wait that runs out writes DT_ERR_TIMEOUT to *d_status and
 * the kernel drains its in-flight copies, frees its tensor memory and
 * returns.  Process-wide setting used by later launches.  Returns DT_OK. */
DT_API int dt_set_wait_limit_ns(int64_t ns);

#ifdef __cplusplus
}
#endif

#endif /* DT_H_ */
