// attn_fused_sm100.cu -- fused partial attention with plan-driven state reuse
// for sm_100a (one persistent kernel; TMA + tcgen05 + TMEM).
//
// What it computes ("DiTango: Cost-Effective Parallel Diffusion Generation
// with Selective Attention State Reuse"):
//   attention state of query rows over KV partition k (Eq. 1-3):
//     OUT = softmax(q K_k^T / sqrt(D)) V_k,  LSE = log sum_j exp(q k_j / sqrt(D))
//   composition of states (Eq. 4), applied over all P partitions of a row;
//   selective compute/reuse (Fig. 6): per (query tile, partition) the plan says
//   COMPUTE (fresh state, written to its cache slot) or REUSE (cached state).
//   With state grouping (grouping of adjacent states) a key set is a group of
//   partitions instead of one, and its slot holds the group's composed state.
// Window mode ("DiTFastAttn: Attention Compression for Diffusion Transformer
// Models", window attention with residual sharing): key sets "window" and
// "complement"; at the anchor step both are computed and R = OUT_full -
// OUT_window is stored, later steps compute the window only and add R.
//
// Work decomposition: a work item is (head, 128-row query tile).  The grid is
// persistent (one CTA per SM) and strides over items head-major so the CTAs
// running together share a head's K/V in L2; each item visits its key sets and
// key tiles in a rotated order so those CTAs do not read the same tile at the
// same moment.  Per CTA, 16 warps (4 warpgroups, registers rebalanced with
// setmaxnreg):
//   warps 0-7   softmax:  two warps per SM sub-partition, each owning 16 rows
//                         of the tile (16-lane TMEM accesses; a thread holds 2
//                         rows x 32 columns).  S (TMEM) -> P (bf16, written back
//                         over S in TMEM), running row max/sum, conditional O
//                         rescale.  Two warps per sub-partition keep the
//                         exponential unit busy while the other warp loads S,
//                         reduces its max or stores P.
//   warps 8-11  epilogue: per reused key set (first, off the critical path):
//                         cached state composed into O_tot (shared memory); per
//                         computed key set: O_part (TMEM) -> registers (O_part
//                         released at once) -> normalised fresh state -> cache
//                         slot, composed into O_tot; per item: O_tot -> O
//                         (bf16), LSE
//   warp 12     MMA QK:   tcgen05.mma S = Q K^T (smem x smem); TMEM alloc/free
//   warp 15     MMA PV:   tcgen05.mma O_part += P V (P from TMEM, V from smem).
//                         Two issuing threads, because one thread issues an
//                         MMA only every ~50 clk: 16 MMAs per 128x128 tile
//                         would nearly fill a single issuer's time.
//   warp 13     TMA:      Q once per item, K tiles into an NS-stage ring
//   warp 14     TMA:      V tiles into an NS-stage ring (released separately
//                         from K: a K stage frees as soon as its QK^T is done)
// Tensor memory (512 columns): three S/P buffers [0,384), O_part [384,384+DP).
// Three buffers let QK^T(g+3) wait only for PV(g), so the chain
// P(g) -> PV(g) -> QK^T(g+3) -> softmax spans three tiles.  O_tot (the
// running composition of an item's states) lives in shared memory, column-
// major fp32, one row per epilogue thread.  DP = head dim padded to a multiple of 16 (72 -> 80):
// a 64-column block uses the 128-byte swizzle, the 16-column tail of D=72 the
// 32-byte swizzle (zero-filled by TMA out-of-bounds handling).
//
// Split-precision PV for the window key set: P = P_hi + P_lo with both halves
// in bf16 (P_lo in the upper half of the S buffer) and two PV MMAs.  The window
// output is later combined with a residual that nearly cancels it, which
// amplifies the relative rounding error of a single bf16 P several times.
//
// Every wait is bounded; a wait that runs out raises an abort flag shared by
// all roles, writes DT_ERR_TIMEOUT to *status, and every role drains its
// in-flight async work before the CTA frees its tensor memory and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/dt.h"
#include "attn_fused.h"
#include "geometry.h"
#include "sm100.cuh"

namespace dt {
namespace {

using namespace sm100;

// 4 warpgroups: softmax (warps 0-7), epilogue (8-11), MMA QK (12) + TMA (13, 14) + MMA PV (15).
constexpr int kThreads = 512;
constexpr int kWarpEpi = 8, kWarpMma = 12, kWarpTmaK = 13, kWarpTmaV = 14, kWarpMmaPV = 15;
// Registers per thread at launch (ptxas: 65536 / 512; the build checks it) and
// the per-warpgroup split after setmaxnreg.  The split must fit the launch
// pool: 128 * (2 * kRegsSoftmax + kRegsEpilogue + kRegsOther) <= kThreads * kLaunchRegs.
constexpr int kLaunchRegs = 128;
constexpr int kRegsSoftmax = 128, kRegsEpilogue = 192, kRegsOther = 64;
static_assert(128 * (2 * kRegsSoftmax + kRegsEpilogue + kRegsOther) <= kThreads * kLaunchRegs, "register split");
constexpr uint64_t kDrainLimitNs = 1000000000ull;   // drains use a fixed limit
constexpr int kMaxDevices = 64;
__device__ __forceinline__ float neg_inf() { return -__int_as_float(0x7f800000); }
#define kNegInf (neg_inf())
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;   // log2 units: rescale O only when the max grows by > 2^8

// Timeline tracing for kernel development (compiled only with -DDT_TRACE):
// CTA 0 records clock64 stamps of each role into a caller-provided buffer.
#ifdef DT_TRACE
__constant__ uint64_t* g_dt_trace = nullptr;   // constant bank: no global load per stamp
#define DT_TR(ev, idx)                                                                             \
  do {                                                                                             \
    if (blockIdx.x == 0 && g_dt_trace && (idx) < 4096)   /* all lanes: no divergence */          \
      g_dt_trace[(ev) * 4096 + (idx)] = clock64();                                                 \
  } while (0)
#else
#define DT_TR(ev, idx) do {} while (0)
#endif

template <int DP>
struct Cfg {
  static constexpr int kN64 = DP / 64;                 // 64-column SW128 blocks
  static constexpr int kTail = (DP % 64) ? 1 : 0;      // one 16-column SW32 block
  static_assert(DP % 64 == 0 || DP % 64 == 16, "padded head dim must be 64k or 64k+16");
  static constexpr int kBlk = 128 * 64 * 2;            // bytes of a 128x64 bf16 block
  static constexpr int kTailBytes = 128 * 16 * 2;      // bytes of a 128x16 bf16 block
  static constexpr int kTileBytes = kN64 * kBlk + kTail * kTailBytes;   // = 128 * DP * 2
  static constexpr int kStages = DP == 128 ? 2 : (DP == 80 ? 4 : 5);
  static constexpr int kNS = 3;                        // S/P buffers in tensor memory
  static constexpr int kColS = 0;
  static constexpr int kColOpart = 128 * kNS;
  static_assert(kColOpart + DP <= 512, "tensor memory budget");
  static constexpr int kOtotBytes = DP * 128 * 4;      // O_tot in shared memory, [128][DP] fp32 (swizzled)
  // barrier indices
  static constexpr int bQFull = 0, bQEmpty = 1, bKFull = 2, bVFull = 2 + kStages, bKEmpty = 2 + 2 * kStages,
                       bVEmpty = 2 + 3 * kStages, bSFull = 2 + 4 * kStages, bPFull = bSFull + kNS,
                       bPVDone = bPFull + kNS, bODSeg = bPVDone + kNS, bOFree = bODSeg + 1, bStFull = bOFree + 1,
                       bStFree = bStFull + 2, bDrain = bStFree + 2, bDrainPV = bDrain + 1, kNumBars = bDrainPV + 1;
  static constexpr int kStatsBytes = 2 * 2 * 128 * 4;
  static constexpr int kSmem = kTileBytes * (1 + 2 * kStages) + kOtotBytes + kStatsBytes + kNumBars * 8 + 16;
  static_assert(kSmem <= 232448, "shared memory budget");
};

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

// A softmax thread holds columns c_j = 8*(j/2) + cq + (j%2), j = 0..31, of
// its rows (increasing in j).  cols_below(x): how many of them are < x;
// cols_in(lo, hi): bit j set iff lo <= c_j <= hi.
__device__ __forceinline__ int cols_below(int x, int cq) {
  const int y = x - cq;
  return imin(imax((y + 7) >> 3, 0), 16) + imin(imax((y + 6) >> 3, 0), 16);
}
__device__ __forceinline__ uint32_t cols_in(int lo, int hi, int cq) {
  const int a = cols_below(lo, cq), b = cols_below(hi + 1, cq);
  const uint32_t upto_b = b >= 32 ? 0xffffffffu : ((1u << b) - 1u);
  const uint32_t upto_a = a >= 32 ? 0xffffffffu : ((1u << a) - 1u);
  return upto_b & ~upto_a;
}
__device__ __forceinline__ uint32_t f2u(float f) { return __float_as_uint(f); }

// Warp-level wait: every lane checks the barrier itself (uniform control
// flow; a lane-0 poll plus broadcast costs a few hundred cycles per wait).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int32_t* status,
                                          uint64_t limit) {
  const bool ok = mbar_wait(bar, parity, abort, status, DT_ERR_TIMEOUT, limit);
  return __all_sync(0xffffffffu, ok);
}

// Plan row of a query tile as a bit mask (bit s set: key set s is COMPUTE).
// Read once per item with independent loads; the plan stays in global
// memory, and testing it byte by byte at every key-set step put a chain of
// dependent loads between consecutive key sets.  At most 64 key sets.
__device__ __forceinline__ uint32_t mask4(uint32_t w) {     // 4 plan bytes (0/1) -> 4 bits
  w &= 0x01010101u;
  return (w | (w >> 7) | (w >> 14) | (w >> 21)) & 0xfu;
}
template <bool WIN>
__device__ __forceinline__ uint64_t plan_mask(const uint8_t* prow, int P) {
  uint64_t m = 0;
  // every loader reads bit 0 of a plan byte (DT_PLAN_COMPUTE = 1, DT_PLAN_REUSE = 0)
  if (WIN) {                                // two key sets
    m = (uint64_t)(prow[0] & 1u) | ((uint64_t)(prow[1] & 1u) << 1);
  } else if ((P & 3) == 0) {                // rows start 4-byte aligned
#pragma unroll 4
    for (int s = 0; s < P; s += 4) m |= (uint64_t)mask4(*reinterpret_cast<const uint32_t*>(prow + s)) << s;
  } else {
    for (int s = 0; s < P; ++s) m |= (uint64_t)(prow[s] & 1u) << s;
  }
  return m;
}
__device__ __forceinline__ bool is_compute(uint64_t cm, int seg) { return (cm >> seg) & 1u; }

template <int MODE>
__device__ __forceinline__ bool item_has_compute(const Geom& G, int qt, uint64_t cm) {
  for (int s = 0; s < G.P; ++s)
    if (is_compute(cm, s) && key_set<MODE>(G, qt, s).ntiles() > 0) return true;
  return false;
}

// Visiting order of the key sets and key tiles of work item idx.  States
// compose associatively and commutatively and the online softmax is order
// free, so any order gives the same result; rotating the start per item keeps
// the CTAs that run together from streaming the same K/V tile at once.
template <bool WIN>
__device__ __forceinline__ int seg_rotation(const Geom& G, int idx) { return WIN ? 0 : idx % G.P; }
template <bool WIN>
__device__ __forceinline__ int visit_seg(const Geom& G, int rot, int j) {
  if (WIN) return j;                          // window set before its complement
  const int s = j + rot;
  return s >= G.P ? s - G.P : s;
}
__device__ __forceinline__ int tile_rotation(int nt, int idx, int seg) { return (idx * 5 + seg * 3) % nt; }
__device__ __forceinline__ int visit_tile(const KeySet& ks, int nt, int off, int i) {
  const int k = i + off;
  return ks.tile(k >= nt ? k - nt : k);
}

// O_tot (the running composition of an item's states, fp32, shared memory):
// row-major [128][DP], its 16-byte chunks XOR-swizzled by (row & 7) inside
// each full group of 8 chunks.  A warp touching one chunk of 32 rows (a row
// per lane) or all chunks of one row (a chunk per lane) then hits every bank
// once per 8-lane phase of a 16-byte access.
template <int DP>
__device__ __forceinline__ float4* ot_chunk(float* sO, int row, int cc) {
  constexpr int kChunks = DP / 4;
  const int sw = ((cc | 7) < kChunks) ? (cc ^ (row & 7)) : cc;
  return reinterpret_cast<float4*>(sO + row * DP + 4 * sw);
}

// Issue O_part += P V for tile g (P read from tensor memory, V from the ring).
template <int DP>
__device__ __forceinline__ bool issue_pv(uint64_t* bars, uint32_t tmem, uint32_t aV, uint32_t g, uint32_t seg,
                                         bool first, bool last, bool precise, volatile int* abort, int32_t* status,
                                         uint64_t lim) {
  using C = Cfg<DP>;
  constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 64 * C::kN64, 0, 1);
  constexpr uint32_t idesc_pvt = idesc_bf16_f32(128, 16, 0, 1);
  const uint32_t sb = g % C::kNS;
  if (!mbar_wait(&bars[C::bPFull + sb], (g / C::kNS) & 1, abort, status, DT_ERR_TIMEOUT, lim)) return false;
  if (first && seg > 0 && !mbar_wait(&bars[C::bOFree], (seg - 1) & 1, abort, status, DT_ERR_TIMEOUT, lim))
    return false;
  const int st = g % C::kStages;
  if (!mbar_wait(&bars[C::bVFull + st], (g / C::kStages) & 1, abort, status, DT_ERR_TIMEOUT, lim)) return false;
  DT_TR(5, g);
  tc_fence_after();
  uint32_t aP = tmem + C::kColS + sb * 128;
  const uint32_t vb = aV + st * C::kTileBytes;
  // 16 keys per MMA; descriptors advance by 16 V rows (2048 bytes in the
  // 128-byte-swizzled blocks, 512 in the 32-byte-swizzled tail)
  uint64_t vd = smem_desc(vb, C::kBlk, 1024, kSwizzle128B);
  uint64_t vdt = smem_desc(vb + C::kN64 * C::kBlk, C::kTailBytes, 256, kSwizzle32B);
  uint32_t acc = first ? 0u : 1u;
#pragma unroll 1
  for (int kk = 0; kk < 8; ++kk) {
    mma_ts(tmem + C::kColOpart, aP, vd, idesc_pv, acc);
    if (C::kTail) mma_ts(tmem + C::kColOpart + 64 * C::kN64, aP, vdt, idesc_pvt, acc);
    if (precise) {                          // P = P_hi + P_lo (P_lo in columns 64..127)
      mma_ts(tmem + C::kColOpart, aP + 64, vd, idesc_pv, 1u);
      if (C::kTail) mma_ts(tmem + C::kColOpart + 64 * C::kN64, aP + 64, vdt, idesc_pvt, 1u);
    }
    acc = 1u;
    aP += 8;
    vd += 2048 >> 4;
    vdt += 512 >> 4;
  }
  mma_commit(&bars[C::bVEmpty + st]);
  mma_commit(&bars[C::bPVDone + sb]);
  if (last) mma_commit(&bars[C::bODSeg]);
  DT_TR(12, g);
  return true;
}

// MODE: key-set mode (kModePartition, kModeWindow, kModeGrouped) in bits 0-1,
// kStateBf16 when the cached OUT is bf16 (partition modes).
constexpr int kStateBf16 = 4;

template <int DP, int MODE>
__global__ void __launch_bounds__(kThreads, 1) attn_partial_fused_kernel(const __grid_constant__ AttnParams p) {
  using C = Cfg<DP>;
  constexpr int KM = MODE & 3;
  constexpr bool WIN = KM == kModeWindow;
  constexpr bool CBF = (MODE & kStateBf16) != 0;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {                       // layout needs 1024-byte alignment
    if (threadIdx.x == 0) atomicCAS(p.status, 0, DT_ERR_UNSUPPORTED);
    return;
  }
  uint8_t* sQ = smem;
  uint8_t* sK = smem + C::kTileBytes;
  uint8_t* sV = sK + C::kStages * C::kTileBytes;
  float* sO = reinterpret_cast<float*>(sV + C::kStages * C::kTileBytes);       // O_tot [128][DP]
  float* stat_m = sO + DP * 128;                                               // [2][128]
  float* stat_l = stat_m + 256;                                                // [2][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(stat_l + 256);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geom& G = p.geom;
  const uint64_t lim = p.wait_limit_ns;

  if (warp == kWarpTmaK && lane == 0) {
    for (int i = 0; i < C::kNumBars; ++i) mbar_init(&bars[i], 1);
    for (int i = 0; i < C::kNS; ++i) mbar_init(&bars[C::bPFull + i], 8 * 32);   // every softmax thread arrives
    // every thread of the arriving role arrives (no single-lane branches)
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[C::bStFull + i], 8 * 32);
      mbar_init(&bars[C::bStFree + i], 4 * 32);
    }
    mbar_init(&bars[C::bOFree], 4 * 32);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async();
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp >= kWarpMma) {
   regs_set<kLaunchRegs, kRegsOther>();
   if (warp == kWarpTmaK || warp == kWarpTmaV) {
    // ------------------------------------------------------------ TMA producers
    // Warp 13 loads Q (once per item) and the K ring, warp 14 the V ring; both
    // walk the same tile sequence.
    if (lane == 0) {
      const bool is_k = warp == kWarpTmaK;
      const CUtensorMap* tm = is_k ? &p.tmK : &p.tmV;
      const CUtensorMap* tmt = is_k ? &p.tmKt : &p.tmVt;
      uint8_t* ring = is_k ? sK : sV;
      uint64_t* full = &bars[is_k ? C::bKFull : C::bVFull];
      uint64_t* empty = &bars[is_k ? C::bKEmpty : C::bVEmpty];
      prefetch_tmap(tm);
      if (C::kTail) prefetch_tmap(tmt);
      if (is_k) { prefetch_tmap(&p.tmQ); if (C::kTail) prefetch_tmap(&p.tmQt); }
      // K/V tiles are re-read by every query tile of the head: keep them in L2
      // against the streaming state-cache traffic; a Q tile is read once.
      const uint64_t pol_keep = l2_policy_evict_last(), pol_once = l2_policy_evict_first();
      uint32_t g = 0, nq = 0;
      for (int idx = p.item0 + blockIdx.x; idx < p.item_end; idx += gridDim.x) {
        const int h = idx / G.nqt, qt = idx - (idx / G.nqt) * G.nqt;
        const uint64_t cm = plan_mask<WIN>(p.plan + (size_t)qt * G.P, G.P);
        const int rot = seg_rotation<WIN>(G, idx);
        if (!item_has_compute<KM>(G, qt, cm)) continue;
        if (is_k) {
          const QTile t = query_tile<KM>(G, qt);
          if (nq > 0 && !mbar_wait(&bars[C::bQEmpty], (nq - 1) & 1, abort_flag, p.status, DT_ERR_TIMEOUT, lim))
            goto tma_done;
          DT_TR(19, nq);
          mbar_arrive_expect_tx(&bars[C::bQFull], C::kTileBytes);
          for (int c = 0; c < C::kN64; ++c)
            tma_load_3d_hint(sQ + c * C::kBlk, &p.tmQ, &bars[C::bQFull], 64 * c, t.q0, h, pol_once);
          if (C::kTail)
            tma_load_3d_hint(sQ + C::kN64 * C::kBlk, &p.tmQt, &bars[C::bQFull], 64 * C::kN64, t.q0, h, pol_once);
          ++nq;
        }
        for (int j = 0; j < G.P; ++j) {
          const int seg = visit_seg<WIN>(G, rot, j);
          if (!is_compute(cm, seg)) continue;
          const KeySet ks = key_set<KM>(G, qt, seg);
          const int nt = ks.ntiles();
          const int toff = nt > 0 ? tile_rotation(nt, idx, seg) : 0;
          for (int i = 0; i < nt; ++i, ++g) {
            const int st = g % C::kStages;
            if (g >= (uint32_t)C::kStages &&
                !mbar_wait(&empty[st], ((g / C::kStages) - 1) & 1, abort_flag, p.status, DT_ERR_TIMEOUT, lim))
              goto tma_done;
            const int row0 = ks.row0(visit_tile(ks, nt, toff, i));
            uint8_t* dst = ring + st * C::kTileBytes;
            DT_TR(is_k ? 8 : 9, g);
            mbar_arrive_expect_tx(&full[st], C::kTileBytes);
            for (int c = 0; c < C::kN64; ++c) tma_load_3d_hint(dst + c * C::kBlk, tm, &full[st], 64 * c, row0, h, pol_keep);
            if (C::kTail) tma_load_3d_hint(dst + C::kN64 * C::kBlk, tmt, &full[st], 64 * C::kN64, row0, h, pol_keep);
          }
        }
      }
    tma_done:
      // let every copy this warp started land before shared memory goes away
      for (int s = 0; s < C::kStages; ++s) {
        if ((uint32_t)s < g) {
          const uint32_t last = g - 1 - ((g - 1 - s) % C::kStages);   // latest tile that used stage s
          volatile int never = 0;
          mbar_wait(&full[s], (last / C::kStages) & 1, &never, p.status, DT_ERR_TIMEOUT, kDrainLimitNs);
        }
      }
      if (is_k && nq > 0) {
        volatile int never = 0;
        mbar_wait(&bars[C::bQFull], (nq - 1) & 1, &never, p.status, DT_ERR_TIMEOUT, kDrainLimitNs);
      }
    }
   } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
      uint32_t g = 0, nq = 0;
      bool ok = true;

      for (int idx = p.item0 + blockIdx.x; idx < p.item_end && ok; idx += gridDim.x) {
        const int qt = idx - (idx / G.nqt) * G.nqt;
        const uint64_t cm = plan_mask<WIN>(p.plan + (size_t)qt * G.P, G.P);
        const int rot = seg_rotation<WIN>(G, idx);
        if (!item_has_compute<KM>(G, qt, cm)) continue;
        if (!mbar_wait(&bars[C::bQFull], nq & 1, abort_flag, p.status, DT_ERR_TIMEOUT, lim)) { ok = false; break; }
        DT_TR(20, nq);
        ++nq;
        tc_fence_after();
        for (int j = 0; j < G.P && ok; ++j) {
          const int seg = visit_seg<WIN>(G, rot, j);
          if (!is_compute(cm, seg)) continue;
          const int nt = key_set<KM>(G, qt, seg).ntiles();
          if (nt == 0) continue;
          for (int i = 0; i < nt; ++i, ++g) {
            const int st = g % C::kStages;
            DT_TR(10, g);
            if (!mbar_wait(&bars[C::bKFull + st], (g / C::kStages) & 1, abort_flag, p.status, DT_ERR_TIMEOUT, lim)) {
              ok = false;
              break;
            }
            // S buffer g%3 held P(g-3): its PV (issued by the PV warp) must be done
            if (g >= (uint32_t)C::kNS &&
                !mbar_wait(&bars[C::bPVDone + g % C::kNS], (g / C::kNS - 1) & 1, abort_flag, p.status,
                           DT_ERR_TIMEOUT, lim)) {
              ok = false;
              break;
            }
            DT_TR(11, g);
            tc_fence_after();
            const uint32_t dS = tmem + C::kColS + (g % C::kNS) * 128;
            const uint32_t kb = aK + st * C::kTileBytes;
            // 16 head-dim columns (32 bytes of each swizzled row) per MMA
            uint32_t acc = 0u;
#pragma unroll 1
            for (int blk = 0; blk < C::kN64; ++blk) {
              uint64_t qd = smem_desc(aQ + blk * C::kBlk, 16, 1024, kSwizzle128B);
              uint64_t kd = smem_desc(kb + blk * C::kBlk, 16, 1024, kSwizzle128B);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                mma_ss(dS, qd, kd, idesc_qk, acc);
                acc = 1u;
                qd += 32 >> 4;
                kd += 32 >> 4;
              }
            }
            if (C::kTail) {
              const uint32_t off = C::kN64 * C::kBlk;
              mma_ss(dS, smem_desc(aQ + off, 16, 256, kSwizzle32B), smem_desc(kb + off, 16, 256, kSwizzle32B),
                     idesc_qk, 1u);
            }
            mma_commit(&bars[C::bSFull + g % C::kNS]);
            mma_commit(&bars[C::bKEmpty + st]);
            DT_TR(0, g);
          }
        }
        mma_commit(&bars[C::bQEmpty]);
      }
      // all MMAs this thread issued complete before tensor memory is freed
      mma_commit(&bars[C::bDrain]);
      volatile int never = 0;
      mbar_wait(&bars[C::bDrain], 0, &never, p.status, DT_ERR_TIMEOUT, kDrainLimitNs);
    }
    __syncwarp();
   } else if (warp == kWarpMmaPV) {
    // ------------------------------------------------------------ PV issuer
    // A second issuing thread: one thread issues a tcgen05.mma only every ~50
    // clk, so QK^T and PV come from separate warps.  Their ordering is explicit:
    // PV(g) waits for P(g); QK^T(g+2) waits for PV(g) through bPVDone.
    if (lane == 0) {
      const uint32_t aV = smem_u32(sV);
      uint32_t g = 0, cseg = 0;
      bool ok = true;
      for (int idx = p.item0 + blockIdx.x; idx < p.item_end && ok; idx += gridDim.x) {
        const int qt = idx - (idx / G.nqt) * G.nqt;
        const uint64_t cm = plan_mask<WIN>(p.plan + (size_t)qt * G.P, G.P);
        const int rot = seg_rotation<WIN>(G, idx);
        if (!item_has_compute<KM>(G, qt, cm)) continue;
        for (int j = 0; j < G.P && ok; ++j) {
          const int seg = visit_seg<WIN>(G, rot, j);
          if (!is_compute(cm, seg)) continue;
          const int nt = key_set<KM>(G, qt, seg).ntiles();
          if (nt == 0) continue;
          for (int i = 0; i < nt && ok; ++i, ++g)
            ok = issue_pv<DP>(bars, tmem, aV, g, cseg, i == 0, i == nt - 1, WIN && seg == 0, abort_flag, p.status,
                              lim);
          ++cseg;
        }
      }
      mma_commit(&bars[C::bDrainPV]);
      volatile int never = 0;
      mbar_wait(&bars[C::bDrainPV], 0, &never, p.status, DT_ERR_TIMEOUT, kDrainLimitNs);
    }
    __syncwarp();
   }
  } else if (warp < kWarpEpi) {
    regs_set<kLaunchRegs, kRegsSoftmax>();
    // ------------------------------------------------------------ softmax
    // Warp w owns tile rows rbase .. rbase+15 (TMEM lanes of its sub-partition
    // w % 4); thread t holds rows ra = rbase + t/4 and rb = ra + 8 at columns
    // 8i + 2(t%4) + {0,1}, i = 0..15.  The P pair of those two columns is P
    // column 4i + t%4, which the 16x128b store writes from the same thread.
    const int rbase = (warp & 3) * 32 + (warp >> 2) * 16;
    const int ra = rbase + (lane >> 2), rb = ra + 8;
    const int cq = 2 * (lane & 3);
    const uint32_t lane_base = static_cast<uint32_t>(rbase) << 16;
    const float sl2 = p.scale_log2;
    uint32_t g = 0, cseg = 0;
    for (int idx = p.item0 + blockIdx.x; idx < p.item_end; idx += gridDim.x) {
      const int qt = idx - (idx / G.nqt) * G.nqt;
      const uint64_t cm = plan_mask<WIN>(p.plan + (size_t)qt * G.P, G.P);
      const int rot = seg_rotation<WIN>(G, idx);
      if (!item_has_compute<KM>(G, qt, cm)) continue;
      const QTile t = query_tile<KM>(G, qt);
      const int qa = t.q0 + ra, qb = t.q0 + rb;
      const int q1 = t.q0 + t.rows - 1;
      for (int j = 0; j < G.P; ++j) {
        const int seg = visit_seg<WIN>(G, rot, j);
        if (!is_compute(cm, seg)) continue;
        const KeySet ks = key_set<KM>(G, qt, seg);
        const int nt = ks.ntiles();
        if (nt == 0) continue;
        const int toff = tile_rotation(nt, idx, seg);
        // running max (log2 units) and partial row sums of rows ra, rb
        float ma = kNegInf, mb = kNegInf;
        uint64_t la[2] = {0ull, 0ull}, lb[2] = {0ull, 0ull};      // packed pairs of partial sums
        const bool precise = WIN && seg == 0;
        for (int i = 0; i < nt; ++i, ++g) {
          const uint32_t sb = g % C::kNS;
          if (warp == 0) DT_TR(15, g);
          if (!warp_wait(&bars[C::bSFull + sb], (g / C::kNS) & 1, abort_flag, p.status, lim)) goto sm_done;
          if (warp == 0) DT_TR(2, g);
          if (warp == 7) DT_TR(14, g);
          tc_fence_after();
          const int tile = visit_tile(ks, nt, toff, i);
          const int k0 = ks.row0(tile);
          const int kvalid = imin(kTile, ks.rowend(tile) - k0);
          const uint32_t sc = tmem + lane_base + C::kColS + sb * 128;
          uint32_t sr[64];
          tmem_ld_16x256b_x8(sc, sr);
          tmem_ld_16x256b_x8(sc + 64, sr + 32);
          tmem_wait_ld();
          if (warp == 0) DT_TR(1, g);
          int mask_kind = 0;   // 1: keep |i-j| <= hw, 2: keep |i-j| > hw
          if (WIN)
            mask_kind = seg == 0 ? (wtile_inside(G, t.q0, q1, tile) ? 0 : 1)
                                 : (wtile_touches(G, t.q0, q1, tile) ? 2 : 0);
          const bool masked = kvalid < kTile || mask_kind != 0;
          if (masked) {
            // kept columns of rows ra and rb as bit masks over this thread's
            // 32 columns (the band |i-j| <= hw is a column interval per row),
            // then one bit test per element: compact code for the edge tiles
            const uint32_t all = cols_in(0, kvalid - 1, cq);
            uint32_t ka = all, kb = all;
            if (mask_kind != 0) {
              const uint32_t wa = cols_in(qa - G.hw - k0, qa + G.hw - k0, cq);
              const uint32_t wb = cols_in(qb - G.hw - k0, qb + G.hw - k0, cq);
              ka = mask_kind == 1 ? (all & wa) : (all & ~wa);
              kb = mask_kind == 1 ? (all & wb) : (all & ~wb);
            }
#pragma unroll
            for (int e = 0; e < 64; ++e) {
              const uint32_t km = (e & 2) ? kb : ka;
              if (!(km & (1u << (2 * (e >> 2) + (e & 1))))) sr[e] = f2u(kNegInf);
            }
          }
          // row maxima: two chains per row, then across the 4 threads of a row
          float xa0 = fmaxf(u2f(sr[0]), u2f(sr[1])), xa1 = fmaxf(u2f(sr[4]), u2f(sr[5]));
          float xb0 = fmaxf(u2f(sr[2]), u2f(sr[3])), xb1 = fmaxf(u2f(sr[6]), u2f(sr[7]));
#pragma unroll
          for (int r4 = 2; r4 < 16; r4 += 2) {
            xa0 = max3f(xa0, u2f(sr[4 * r4]), u2f(sr[4 * r4 + 1]));
            xa1 = max3f(xa1, u2f(sr[4 * r4 + 4]), u2f(sr[4 * r4 + 5]));
            xb0 = max3f(xb0, u2f(sr[4 * r4 + 2]), u2f(sr[4 * r4 + 3]));
            xb1 = max3f(xb1, u2f(sr[4 * r4 + 6]), u2f(sr[4 * r4 + 7]));
          }
          float mxa = fmaxf(xa0, xa1), mxb = fmaxf(xb0, xb1);
          mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 1));
          mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 1));
          mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 2));
          mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 2));
          if (warp == 0) DT_TR(3, g);
          const float mxa2 = mxa * sl2, mxb2 = mxb * sl2;
          const float na = (i == 0) ? mxa2 : ((mxa2 > ma + kRescaleThreshold) ? mxa2 : ma);
          const float nb = (i == 0) ? mxb2 : ((mxb2 > mb + kRescaleThreshold) ? mxb2 : mb);
          // a row that has seen only masked keys (max -inf) has O_part = 0 and
          // l = 0: it takes the new reference without a rescale (and without
          // waiting for the previous PV)
          const bool resa = (i > 0) && (na != ma) && (ma != kNegInf);
          const bool resb = (i > 0) && (nb != mb) && (mb != kNegInf);
          if (__any_sync(0xffffffffu, resa || resb)) {
            // O_part holds the previous tiles' sum: wait for its last PV, then rescale
            if (!warp_wait(&bars[C::bPVDone + (g - 1) % C::kNS], ((g - 1) / C::kNS) & 1, abort_flag, p.status, lim))
              goto sm_done;
            tc_fence_after();
            const float alpha_a = resa ? ex2(ma - na) : 1.f, alpha_b = resb ? ex2(mb - nb) : 1.f;
            const uint32_t oc = tmem + lane_base + C::kColOpart;
#pragma unroll 1
            for (int c0 = 0; c0 < DP; c0 += 16) {
              uint32_t o[8];
              tmem_ld_16x256b_x2(oc + c0, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 8; ++e) o[e] = f2u(u2f(o[e]) * ((e & 2) ? alpha_b : alpha_a));
              tmem_st_16x256b_x2(oc + c0, o);
            }
            tmem_wait_st();
            const uint64_t aa = pk2(alpha_a, alpha_a), ab = pk2(alpha_b, alpha_b);
#pragma unroll
            for (int k = 0; k < 2; ++k) { la[k] = fma2(la[k], aa, 0ull); lb[k] = fma2(lb[k], ab, 0ull); }
          }
          ma = na; mb = nb;
          const float mra = (ma == kNegInf) ? 0.f : ma, mrb = (mb == kNegInf) ? 0.f : mb;
          const uint64_t sl2x2 = pk2(sl2, sl2), nma = pk2(-mra, -mra), nmb = pk2(-mrb, -mrb);
          // exponentials, 8 repetitions (32 P columns) per TMEM store
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            uint32_t ph[16];
#pragma unroll
            for (int r4 = 0; r4 < 8; ++r4) {
              const int e = 4 * (8 * hf + r4);
              float x0, x1, x2, x3;
              upk2(fma2(pk2(u2f(sr[e]), u2f(sr[e + 1])), sl2x2, nma), x0, x1);
              upk2(fma2(pk2(u2f(sr[e + 2]), u2f(sr[e + 3])), sl2x2, nmb), x2, x3);
              const float p0 = ex2(x0), p1 = ex2(x1), p2 = ex2(x2), p3 = ex2(x3);
              la[r4 & 1] = add2(la[r4 & 1], pk2(p0, p1));
              lb[r4 & 1] = add2(lb[r4 & 1], pk2(p2, p3));
              ph[2 * r4] = pack_bf16x2(p0, p1);
              ph[2 * r4 + 1] = pack_bf16x2(p2, p3);
              if (precise) {                      // bf16 residuals overwrite the consumed logits
                sr[e] = pack_bf16x2(p0 - u2f(ph[2 * r4] << 16), p1 - u2f(ph[2 * r4] & 0xffff0000u));
                sr[e + 1] = pack_bf16x2(p2 - u2f(ph[2 * r4 + 1] << 16), p3 - u2f(ph[2 * r4 + 1] & 0xffff0000u));
              }
            }
            tmem_st_16x128b_x8(sc + 32 * hf, ph);
            if (precise) {                        // P_lo in columns 64..127
              uint32_t pl[16];
#pragma unroll
              for (int r4 = 0; r4 < 8; ++r4) {
                pl[2 * r4] = sr[4 * (8 * hf + r4)];
                pl[2 * r4 + 1] = sr[4 * (8 * hf + r4) + 1];
              }
              tmem_st_16x128b_x8(sc + 64 + 32 * hf, pl);
            }
          }
          if (warp == 0) DT_TR(6, g);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&bars[C::bPFull + sb]);      // all lanes: no divergent single-lane branch per tile
          if (warp == 0) DT_TR(4, g);
          if (warp == 7) DT_TR(13, g);
        }
        {
          float sa, sbm;
          {
            float u0, u1, v0, v1;
            upk2(add2(la[0], la[1]), u0, u1);
            upk2(add2(lb[0], lb[1]), v0, v1);
            sa = u0 + u1;
            sbm = v0 + v1;
          }
          sa += __shfl_xor_sync(0xffffffffu, sa, 1);
          sbm += __shfl_xor_sync(0xffffffffu, sbm, 1);
          sa += __shfl_xor_sync(0xffffffffu, sa, 2);
          sbm += __shfl_xor_sync(0xffffffffu, sbm, 2);
          const uint32_t st = cseg & 1;
          if (cseg >= 2 && !warp_wait(&bars[C::bStFree + st], ((cseg >> 1) - 1) & 1, abort_flag, p.status, lim))
            goto sm_done;
          // the 4 threads of a row hold the same values: all of them write
          stat_m[st * 128 + ra] = ma;
          stat_l[st * 128 + ra] = sa;
          stat_m[st * 128 + rb] = mb;
          stat_l[st * 128 + rb] = sbm;
          mbar_arrive(&bars[C::bStFull + st]);
          ++cseg;
        }
      }
    }
  sm_done:;
  } else {
    regs_set<kLaunchRegs, kRegsEpilogue>();
    // ------------------------------------------------------------ epilogue
    const int q4 = warp - kWarpEpi;
    const int r = q4 * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t opart = tmem + lane_base + C::kColOpart;
    constexpr int D = DP == 80 ? 72 : DP;   // head dims 64, 72, 128 (padded 64, 80, 128)
    // O_tot rows are unnormalised relative to m_tot.  A thread owns its row
    // (fresh states, output); the reuse merge updates the warp's 32 rows
    // cooperatively, one row per load instruction.
    uint32_t cseg = 0;
    uint32_t n_comp = 0, n_skip = 0, n_fresh = 0, n_read = 0;
    for (int idx = p.item0 + blockIdx.x; idx < p.item_end; idx += gridDim.x) {
      const int h = idx / G.nqt, qt = idx - (idx / G.nqt) * G.nqt;
      const uint64_t cm = plan_mask<WIN>(p.plan + (size_t)qt * G.P, G.P);
      const int rot = seg_rotation<WIN>(G, idx);
      const QTile t = query_tile<KM>(G, qt);
      const int qrow = t.q0 + r;
      const bool valid = r < t.rows;
      float m_tot = kNegInf, l_tot = 0.f;
      bool have = false, use_r = false;
      // O_tot starts at zero, so the merges below need no separate first-state case
#pragma unroll 4
      for (int cc = 0; cc < DP / 4; ++cc) *ot_chunk<DP>(sO, r, cc) = make_float4(0.f, 0.f, 0.f, 0.f);
      __syncwarp();
      // Cached states of the REUSE pairs are composed into O_tot interleaved
      // with the fresh ones, a fixed share after each fresh state, once its
      // O_part is back with the MMA warps (their loads are latency-bound;
      // composing them before a fresh state would hold up the release of
      // O_part that the next key set's PV waits on).  The order depends
      // only on the plan, so results are reproducible run to run.  jr walks
      // the key sets in visiting order; merged counts reused sets done.
      const int sets_fresh = __popcll(cm), sets_reused = G.P - sets_fresh;
      int jr = 0, merged = 0, fi = 0;
      auto merge_next_reused = [&]() {
        for (; jr < G.P; ++jr) {
          const int seg = visit_seg<WIN>(G, rot, jr);
          if (is_compute(cm, seg)) continue;
          n_skip += counted_blocks<KM>(G, qt, seg);   // same in every lane; thread 0 reports
          ++n_read;
          if (WIN) { use_r = true; ++merged; continue; }   // complement reused: add R at the end
          if (warp == kWarpEpi) DT_TR(17, n_read);
          const size_t slot = ((size_t)seg * G.H + h) * G.S + qrow;
          // The warp's 32 slot rows are contiguous: lane l reads 16 bytes (8
          // of bf16) of every row, so each load instruction covers one whole
          // row.  All 32 rows and the rows' LSEs are loaded together (one
          // memory round trip); rows past a ragged tile are not read, and
          // rows whose state is empty (LSE -inf) are zeroed after the load.
          const size_t row0 = slot - r + 32 * q4;           // slot row of the warp's first row
          const bool lane_on = 4 * lane < D;
          const uint32_t vrows = __ballot_sync(0xffffffffu, valid);
          const float lse_c = valid ? __ldcs(p.cache_L + slot) : kNegInf;
          float4 cv[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const bool on = lane_on && ((vrows >> k) & 1u);
            if (CBF) {
              const uint2 hv = on ? __ldcs(reinterpret_cast<const uint2*>(
                                        reinterpret_cast<const __nv_bfloat16*>(p.cache_O) + (row0 + k) * D) + lane)
                                  : make_uint2(0, 0);
              cv[k] = make_float4(bf16lo(hv.x), bf16hi(hv.x), bf16lo(hv.y), bf16hi(hv.y));
            } else {
              cv[k] = on ? __ldcs(reinterpret_cast<const float4*>(p.cache_O + (row0 + k) * D) + lane)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
            }
          }
          const bool nonempty = lse_c > kNegInf;
          const float m_c = lse_c * kLog2e;
          float a, b, m_new;
          if (!have) { m_new = m_c; a = 0.f; b = nonempty ? 1.f : 0.f; }
          else {
            m_new = nonempty ? fmaxf(m_tot, m_c) : m_tot;
            a = ex2(m_tot - m_new);
            b = nonempty ? ex2(m_c - m_new) : 0.f;
          }
          const float l_new = a * l_tot + b;
          const uint32_t live = __ballot_sync(0xffffffffu, valid && nonempty);
          __syncwarp();                                   // the lanes' own-row writes are visible
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const int row = 32 * q4 + k;
            const float ak = __shfl_sync(0xffffffffu, a, k), bk = __shfl_sync(0xffffffffu, b, k);
            if (lane_on) {
              const float4 c = ((live >> k) & 1u) ? cv[k] : make_float4(0.f, 0.f, 0.f, 0.f);
              float4* o = ot_chunk<DP>(sO, row, lane);
              float4 ov = *o;
              ov.x = fmaf(ak, ov.x, bk * c.x);
              ov.y = fmaf(ak, ov.y, bk * c.y);
              ov.z = fmaf(ak, ov.z, bk * c.z);
              ov.w = fmaf(ak, ov.w, bk * c.w);
              *o = ov;
            }
          }
          __syncwarp();
          if (have || nonempty) { m_tot = m_new; l_tot = l_new; }
          have = have || nonempty;
          ++jr;
          ++merged;
          if (warp == kWarpEpi) DT_TR(18, n_read);
          return;
        }
      };
      // (2) fresh states, in the order the MMA produces them
      for (int j = 0; j < G.P; ++j) {
        const int seg = visit_seg<WIN>(G, rot, j);
        if (!is_compute(cm, seg)) continue;
        const int nt = key_set<KM>(G, qt, seg).ntiles();
        const size_t slot = ((size_t)seg * G.H + h) * G.S + qrow;
        n_comp += counted_blocks<KM>(G, qt, seg);
        ++n_fresh;
        if (nt == 0) {             // empty key set: the identity state
          if (WIN && valid && seg == 1) {
            // empty complement (the band covers every key of the row's
            // tile): full attention equals window attention, so R = 0
            float4* dst = reinterpret_cast<float4*>(p.R + ((size_t)h * G.S + qrow) * D);
            for (int d = 0; d < D / 4; ++d) __stcs(dst + d, make_float4(0.f, 0.f, 0.f, 0.f));
          }
          if (!WIN && valid) {
            if (CBF) {
              uint2* dst = reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(p.cache_O) + slot * D);
              for (int d = 0; d < D / 4; ++d) __stcs(dst + d, make_uint2(0, 0));
            } else {
              float4* dst = reinterpret_cast<float4*>(p.cache_O + slot * D);
              for (int d = 0; d < D / 4; ++d) __stcs(dst + d, make_float4(0.f, 0.f, 0.f, 0.f));
            }
            __stcs(p.cache_L + slot, kNegInf);
          }
          continue;
        }
        const uint32_t st = cseg & 1;
        ++fi;
        if (!warp_wait(&bars[C::bStFull + st], (cseg >> 1) & 1, abort_flag, p.status, lim)) goto ep_done;
        const float m_s = stat_m[st * 128 + r], l_s = stat_l[st * 128 + r];
        mbar_arrive(&bars[C::bStFree + st]);
        if (!warp_wait(&bars[C::bODSeg], cseg & 1, abort_flag, p.status, lim)) goto ep_done;
        if (warp == kWarpEpi) DT_TR(21, cseg);
        tc_fence_after();
        // O_part -> registers, then hand O_part straight back to the MMA warps
        uint32_t op[DP];
#pragma unroll
        for (int c0 = 0; c0 < DP; c0 += 16) tmem_ld16p(opart + c0, op + c0);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&bars[C::bOFree]);
        if (warp == kWarpEpi) DT_TR(7, cseg);
        const bool nonempty = l_s > 0.f;
        const float inv_l = nonempty ? 1.f / l_s : 0.f;
        float a, b, m_new;
        if (!have) { m_new = m_s; a = 0.f; b = nonempty ? 1.f : 0.f; }
        else {
          m_new = nonempty ? fmaxf(m_tot, m_s) : m_tot;
          a = ex2(m_tot - m_new);
          b = nonempty ? ex2(m_s - m_new) : 0.f;
        }
        const float l_new = a * l_tot + b * l_s;
        const bool make_r = WIN && seg == 1;
        const float inv_tot = (have && l_tot > 0.f) ? 1.f / l_tot : 0.f;
        const float inv_new = l_new > 0.f ? 1.f / l_new : 0.f;
        // state error of this key set (anchor-guided planning): the slot's
        // previous OUT is read before it is overwritten
        const bool track = !WIN && p.err != nullptr &&
                           (p.err_all || seg == (KM == kModeGrouped ? 0 : query_tile<KM>(G, qt).part));
        float e_diff = 0.f, e_norm = 0.f;
        // 8 columns per step (D = 64, 72, 128 are multiples of 8): two O_tot
        // chunks, one 32-byte store of the fresh fp32 state when the cache is
        // 32-byte aligned (rows are D * 4 bytes, a multiple of 32), one 16-byte
        // store of a bf16 state
#pragma unroll
        for (int c = 0; c < D; c += 8) {
          float old[8], nw[8], x[8];
          float4* oc0 = ot_chunk<DP>(sO, r, c / 4);
          float4* oc1 = ot_chunk<DP>(sO, r, c / 4 + 1);
          const float4 o0 = *oc0, o1 = *oc1;
          old[0] = o0.x; old[1] = o0.y; old[2] = o0.z; old[3] = o0.w;
          old[4] = o1.x; old[5] = o1.y; old[6] = o1.z; old[7] = o1.w;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            x[k] = u2f(op[c + k]);
            nw[k] = fmaf(a, old[k], b * x[k]);
          }
          *oc0 = make_float4(nw[0], nw[1], nw[2], nw[3]);
          *oc1 = make_float4(nw[4], nw[5], nw[6], nw[7]);
          if (valid && track) {
            float ov[8];
            if (CBF) {
              const uint4 hv = __ldcs(reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.cache_O) + slot * D + c));
              ov[0] = bf16lo(hv.x); ov[1] = bf16hi(hv.x); ov[2] = bf16lo(hv.y); ov[3] = bf16hi(hv.y);
              ov[4] = bf16lo(hv.z); ov[5] = bf16hi(hv.z); ov[6] = bf16lo(hv.w); ov[7] = bf16hi(hv.w);
            } else {
              const float4 v0 = __ldcs(reinterpret_cast<const float4*>(p.cache_O + slot * D + c));
              const float4 v1 = __ldcs(reinterpret_cast<const float4*>(p.cache_O + slot * D + c + 4));
              ov[0] = v0.x; ov[1] = v0.y; ov[2] = v0.z; ov[3] = v0.w;
              ov[4] = v1.x; ov[5] = v1.y; ov[6] = v1.z; ov[7] = v1.w;
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const float nv = x[k] * inv_l;
              e_diff = fmaf(nv - ov[k], nv - ov[k], e_diff);
              e_norm = fmaf(nv, nv, e_norm);
            }
          }
          if (valid) {
            if (!WIN && CBF) {
              uint4 pk;
              pk.x = pack_bf16x2(x[0] * inv_l, x[1] * inv_l);
              pk.y = pack_bf16x2(x[2] * inv_l, x[3] * inv_l);
              pk.z = pack_bf16x2(x[4] * inv_l, x[5] * inv_l);
              pk.w = pack_bf16x2(x[6] * inv_l, x[7] * inv_l);
              __stcs(reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.cache_O) + slot * D + c), pk);
            } else if (!WIN) {
              const float4 f0 = make_float4(x[0] * inv_l, x[1] * inv_l, x[2] * inv_l, x[3] * inv_l);
              const float4 f1 = make_float4(x[4] * inv_l, x[5] * inv_l, x[6] * inv_l, x[7] * inv_l);
              float* dst = p.cache_O + slot * D + c;
              if (p.cache_v8) {
                st_cs_v8(dst, f0, f1);
              } else {
                __stcs(reinterpret_cast<float4*>(dst), f0);
                __stcs(reinterpret_cast<float4*>(dst + 4), f1);
              }
            } else if (make_r) {
              float* dst = p.R + ((size_t)h * G.S + qrow) * D + c;
              __stcs(reinterpret_cast<float4*>(dst), make_float4(nw[0] * inv_new - old[0] * inv_tot,
                                                                nw[1] * inv_new - old[1] * inv_tot,
                                                                nw[2] * inv_new - old[2] * inv_tot,
                                                                nw[3] * inv_new - old[3] * inv_tot));
              __stcs(reinterpret_cast<float4*>(dst + 4), make_float4(nw[4] * inv_new - old[4] * inv_tot,
                                                                    nw[5] * inv_new - old[5] * inv_tot,
                                                                    nw[6] * inv_new - old[6] * inv_tot,
                                                                    nw[7] * inv_new - old[7] * inv_tot));
            }
          }
        }
        if (track) {
          // sums over the warp's 32 rows, then one entry per (tile, set, head, warp)
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            e_diff += __shfl_xor_sync(0xffffffffu, e_diff, o);
            e_norm += __shfl_xor_sync(0xffffffffu, e_norm, o);
          }
          if (lane == 0) {
            float* e2 = p.err + ((((size_t)qt * G.P + seg) * G.H + h) * 4 + q4) * 2;
            e2[0] = e_diff;
            e2[1] = e_norm;
          }
        }
        if (!WIN && valid) __stcs(p.cache_L + slot, nonempty ? (m_s + lg2(l_s)) * kLn2 : kNegInf);
        if (warp == kWarpEpi) DT_TR(22, cseg);
        if (have || nonempty) { m_tot = m_new; l_tot = l_new; }
        have = have || nonempty;
        ++cseg;
        // this fresh state's share of the cached states, composed while the
        // MMA warps compute the next key set (O_part is already released)
        while (jr < G.P && merged * sets_fresh < fi * sets_reused) merge_next_reused();
      }
      while (jr < G.P) merge_next_reused();
      // final: O = O_tot / l_tot (+ R), LSE = m_tot + log2(l_tot), in natural units
      if (valid) {
        const float inv = (have && l_tot > 0.f) ? 1.f / l_tot : 0.f;
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.O) + ((size_t)h * G.S + qrow) * D;
        if (WIN && use_r) {
          // the residual row is read whole before any output store (one
          // memory round trip); 8 output columns (16 bytes of bf16) per store
          const float4* rr = reinterpret_cast<const float4*>(p.R + ((size_t)h * G.S + qrow) * D);
          float4 rv[D / 4];
#pragma unroll
          for (int c = 0; c < D / 4; ++c) rv[c] = __ldcs(rr + c);
#pragma unroll
          for (int c = 0; c < D; c += 8) {
            const float4 o0 = *ot_chunk<DP>(sO, r, c / 4), o1 = *ot_chunk<DP>(sO, r, c / 4 + 1);
            const float4 r0 = rv[c / 4], r1 = rv[c / 4 + 1];
            uint4 pk;
            pk.x = pack_bf16x2(fmaf(o0.x, inv, r0.x), fmaf(o0.y, inv, r0.y));
            pk.y = pack_bf16x2(fmaf(o0.z, inv, r0.z), fmaf(o0.w, inv, r0.w));
            pk.z = pack_bf16x2(fmaf(o1.x, inv, r1.x), fmaf(o1.y, inv, r1.y));
            pk.w = pack_bf16x2(fmaf(o1.z, inv, r1.z), fmaf(o1.w, inv, r1.w));
            __stcs(reinterpret_cast<uint4*>(dst + c), pk);
          }
        } else {   // 8 output columns (16 bytes of bf16) per store
#pragma unroll 2
          for (int c = 0; c < D; c += 8) {
            const float4 o0 = *ot_chunk<DP>(sO, r, c / 4), o1 = *ot_chunk<DP>(sO, r, c / 4 + 1);
            uint4 pk;
            pk.x = pack_bf16x2(o0.x * inv, o0.y * inv);
            pk.y = pack_bf16x2(o0.z * inv, o0.w * inv);
            pk.z = pack_bf16x2(o1.x * inv, o1.y * inv);
            pk.w = pack_bf16x2(o1.z * inv, o1.w * inv);
            __stcs(reinterpret_cast<uint4*>(dst + c), pk);
          }
        }
        __stcs(p.L + (size_t)h * G.S + qrow, (have && l_tot > 0.f) ? (m_tot + lg2(l_tot)) * kLn2 : kNegInf);
      }
      if (warp == kWarpEpi) DT_TR(16, (idx - p.item0) / gridDim.x);
    }
  ep_done:
    if (r == 0 && p.counters) {
      atomicAdd(reinterpret_cast<unsigned long long*>(p.counters + 0), (unsigned long long)n_comp);
      atomicAdd(reinterpret_cast<unsigned long long*>(p.counters + 1), (unsigned long long)n_skip);
      atomicAdd(reinterpret_cast<unsigned long long*>(p.counters + 2), (unsigned long long)n_fresh);
      atomicAdd(reinterpret_cast<unsigned long long*>(p.counters + 3), (unsigned long long)n_read);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int DP, int MODE>
int launch_dp(const AttnParams& kp, int grid, cudaStream_t stream) {
  using C = Cfg<DP>;
  // The shared-memory attribute belongs to the function on each device: set
  // it once per device (a repeated set from racing threads is harmless).
  static std::atomic<bool> attr_set[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DT_ERR_CUDA;
  const bool cached = dev >= 0 && dev < kMaxDevices;
  if (!cached || !attr_set[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(attn_partial_fused_kernel<DP, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmem) != cudaSuccess)
      return DT_ERR_CUDA;
    if (cached) attr_set[dev].store(true, std::memory_order_release);
  }
  attn_partial_fused_kernel<DP, MODE><<<grid, kThreads, C::kSmem, stream>>>(kp);
  return cudaGetLastError() == cudaSuccess ? DT_OK : DT_ERR_CUDA;
}

}  // namespace

#ifdef DT_TRACE
extern "C" __attribute__((visibility("default"))) int dt_debug_trace_set(uint64_t* d_buf) {
  return cudaMemcpyToSymbol(g_dt_trace, &d_buf, sizeof(d_buf)) == cudaSuccess ? 0 : -4;
}
#endif

int attn_fused_smem_bytes(int dp) {
  switch (dp) {
    case 64: return Cfg<64>::kSmem;
    case 80: return Cfg<80>::kSmem;
    case 128: return Cfg<128>::kSmem;
  }
  return -1;
}

template <int DP>
int launch_mode(const AttnParams& kp, int grid, cudaStream_t stream) {
  if (kp.window > 0) return launch_dp<DP, kModeWindow>(kp, grid, stream);
  if (kp.geom.grp > 0)
    return kp.state_bf16 ? launch_dp<DP, kModeGrouped | kStateBf16>(kp, grid, stream)
                         : launch_dp<DP, kModeGrouped>(kp, grid, stream);
  return kp.state_bf16 ? launch_dp<DP, kModePartition | kStateBf16>(kp, grid, stream)
                       : launch_dp<DP, kModePartition>(kp, grid, stream);
}

int launch_attn_fused(const AttnParams& kp, int dp, int grid, cudaStream_t stream) {
  switch (dp) {
    case 64: return launch_mode<64>(kp, grid, stream);
    case 80: return launch_mode<80>(kp, grid, stream);
    case 128: return launch_mode<128>(kp, grid, stream);
  }
  return DT_ERR_UNSUPPORTED;
}

}  // namespace dt
