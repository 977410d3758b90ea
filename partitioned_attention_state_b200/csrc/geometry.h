// geometry.h -- partition, query-tile and key-tile geometry shared by the host
// plan builder and the device kernels of libdt.
//
// Context partitioning ("DiTango", the sequence is split into P contiguous
// partitions): c = ceil(S/P), partition k = [k*c, min((k+1)*c, S)).  Query and
// key tiles are 128 rows and partition-local, so the last tile of a partition
// may be short and no tile straddles two partitions.
//
// Window mode ("DiTFastAttn", window attention): key j is inside query i's
// window iff |i - j| <= W/2 on the flattened token order; query tiles and key
// tiles then run over the whole sequence.  A query tile has two key sets:
//   set 0 "window":     key tiles touching the band, masked to |i-j| <= W/2;
//   set 1 "complement": every key tile not fully inside the band, masked to
//                       |i-j| > W/2.
// Key tiles that straddle the band edge belong to both sets (with opposite
// masks), so the two sets partition the (query, key) pairs exactly.
//
// State grouping ("DiTango", grouping of spatially adjacent states, group size
// g >= 1): the partitions form m = ceil(P/g) groups G_i = [i g, min((i+1)g, P)).
// A query tile of partition q has 1 + m key sets: set 0 is {q} (the local
// state, handled separately) and set 1 + i is G_i without q, so the group that
// holds q keeps g - 1 partitions.  The tiles of a grouped set are the
// partition-local tiles of its partitions in increasing partition order.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define DT_HD __host__ __device__ __forceinline__
#else
#define DT_HD inline
#endif

namespace dt {

constexpr int kTile = 128;

DT_HD int ceil_div(int a, int b) { return (a + b - 1) / b; }
DT_HD int imin(int a, int b) { return a < b ? a : b; }
DT_HD int imax(int a, int b) { return a > b ? a : b; }

struct Geom {
  int H, S, D, P;      // P = number of key sets per query tile (2 in window mode)
  int window;          // W (window mode) or 0
  int c;               // partition length (partition modes)
  int tpp;             // query tiles per full partition (partition modes)
  int nqt;             // query tiles per head
  int nkt;             // key tiles over the whole sequence (window mode)
  int hw;              // W / 2
  int parts;           // partitions (partition modes)
  int grp;             // group size g of grouped key sets, 0 = one key set per partition
  int kl, tl;          // last non-empty partition and its key tiles (grouped sets)
};

DT_HD Geom make_geom(int H, int S, int D, int P, int window, int group = 0) {
  Geom g;
  g.H = H; g.S = S; g.D = D; g.window = window;
  g.hw = window / 2;
  g.grp = 0;
  g.kl = g.tl = 0;
  if (window > 0) {
    g.P = 2;
    g.parts = 1;
    g.c = S;
    g.tpp = ceil_div(S, kTile);
    g.nqt = g.tpp;
    g.nkt = g.tpp;
  } else {
    g.parts = P;
    g.grp = group > 0 ? group : 0;
    g.P = group > 0 ? 1 + ceil_div(P, group) : P;
    g.c = S > 0 ? ceil_div(S, P) : 0;
    g.tpp = ceil_div(g.c, kTile);
    if (S > 0) {
      g.kl = ceil_div(S, g.c) - 1;
      g.tl = ceil_div(S - g.kl * g.c, kTile);
    }
    // partitions 0..kl-1 are full (c rows); the last non-empty one may be short
    int nq = 0;
    for (int k = 0; k < g.parts; ++k) {
      int a = imin(k * g.c, S), b = imin((k + 1) * g.c, S);
      nq += ceil_div(b - a, kTile);
    }
    g.nqt = nq;
    g.nkt = ceil_div(S, kTile);
  }
  return g;
}

// Mode of a geometry call: W = 0 partition mode (one key set per partition),
// 1 window mode, 2 grouped key sets, -1 read from g.window and g.grp at run
// time.  Kernels instantiate the mode they run so that the other modes' code
// is not compiled into them.
constexpr int kModePartition = 0, kModeWindow = 1, kModeGrouped = 2;
template <int W>
DT_HD bool is_window(const Geom& g) { return W < 0 ? g.window > 0 : W == kModeWindow; }
template <int W>
DT_HD bool is_grouped(const Geom& g) { return W < 0 ? (g.window == 0 && g.grp > 0) : W == kModeGrouped; }

DT_HD int part_begin(const Geom& g, int k) { return imin(k * g.c, g.S); }
DT_HD int part_end(const Geom& g, int k) { return imin((k + 1) * g.c, g.S); }

// Query tile qt -> (partition, first row, rows).
struct QTile { int part, q0, rows; };

template <int W = -1>
DT_HD QTile query_tile(const Geom& g, int qt) {
  QTile t;
  if (is_window<W>(g)) {
    t.part = 0;
    t.q0 = qt * kTile;
    t.rows = imin(kTile, g.S - t.q0);
  } else {
    t.part = qt / g.tpp;
    int j = qt - t.part * g.tpp;
    t.q0 = part_begin(g, t.part) + j * kTile;
    t.rows = imin(kTile, part_end(g, t.part) - t.q0);
  }
  return t;
}

// Window-band relations of a query tile [q0, q1] (inclusive) and key tile t.
DT_HD bool wtile_touches(const Geom& g, int q0, int q1, int t) {
  int a = t * kTile, b = imin(a + kTile, g.S) - 1;
  return (a - q1 <= g.hw) && (q0 - b <= g.hw);
}
DT_HD bool wtile_inside(const Geom& g, int q0, int q1, int t) {
  int a = t * kTile, b = imin(a + kTile, g.S) - 1;
  return (b - q0 <= g.hw) && (q1 - a <= g.hw);
}

// Key tiles of key set `seg` for query tile `qt`: at most two contiguous
// ranges of tile indices [r0b, r0e) and [r1b, r1e), tiles indexed relative to
// `base` (first key row of tile 0 of the set) and clipped to `kend` (one past
// the set's last key row).
//
// A grouped set (tpp > 0) has one range [0, ntiles): tile t is local tile
// t % tpp of the (t / tpp)-th partition of the list pa, pa+1, ... that skips
// partition `skip`.  Every listed partition before the last non-empty one of
// the sequence is full (tpp tiles), so the division finds the partition.
struct KeySet {
  int base, kend;
  int r0b, r0e, r1b, r1e;
  int tpp, pa, skip, c, S;   // grouped sets only (tpp = 0 otherwise)
  DT_HD int ntiles() const { return (r0e - r0b) + (r1e - r1b); }
  // i-th tile of the set (0 <= i < ntiles) -> tile index
  DT_HD int tile(int i) const { return i < (r0e - r0b) ? r0b + i : r1b + (i - (r0e - r0b)); }
  // first key row of tile t, and one past the last key row its partition holds
  DT_HD int row0(int t) const {
    if (tpp == 0) return base + t * kTile;
    const int j = t / tpp;
    const int pk = pa + j + (pa + j >= skip ? 1 : 0);
    return pk * c + (t - j * tpp) * kTile;
  }
  DT_HD int rowend(int t) const {
    if (tpp == 0) return kend;
    const int j = t / tpp;
    const int pk = pa + j + (pa + j >= skip ? 1 : 0);
    return imin((pk + 1) * c, S);
  }
};

// Key tiles of grouped key set `seg` of a query tile in partition q.
DT_HD KeySet grouped_key_set(const Geom& g, int q, int seg) {
  KeySet ks;
  ks.r1b = ks.r1e = 0;
  ks.r0b = 0;
  if (seg == 0) {                       // the local partition
    ks.tpp = 0;
    ks.base = part_begin(g, q);
    ks.kend = part_end(g, q);
    ks.r0e = ceil_div(ks.kend - ks.base, kTile);
    return ks;
  }
  const int a = (seg - 1) * g.grp, b = imin(seg * g.grp, g.parts);
  const bool has_q = a <= q && q < b;
  ks.tpp = g.tpp > 0 ? g.tpp : 1;
  ks.pa = a;
  ks.skip = has_q ? q : 0x7fffffff;
  ks.c = g.c;
  ks.S = g.S;
  ks.base = part_begin(g, a);
  ks.kend = part_end(g, b - 1);
  // full partitions of the list (below the last non-empty one), then that one
  const int fb = imin(b, g.kl);
  int nfull = imax(0, fb - a) - ((has_q && q < fb) ? 1 : 0);
  int nt = nfull * g.tpp;
  if (g.S > 0 && a <= g.kl && g.kl < b && q != g.kl) nt += g.tl;
  ks.r0e = nt;
  return ks;
}

template <int W = -1>
DT_HD KeySet key_set(const Geom& g, int qt, int seg) {
  KeySet ks;
  if (!is_window<W>(g)) {
    if (is_grouped<W>(g)) return grouped_key_set(g, query_tile<W>(g, qt).part, seg);
    ks.tpp = 0;
    ks.base = part_begin(g, seg);
    ks.kend = part_end(g, seg);
    ks.r0b = 0; ks.r0e = ceil_div(ks.kend - ks.base, kTile);
    ks.r1b = ks.r1e = 0;
    return ks;
  }
  ks.tpp = 0;
  QTile t = query_tile<W>(g, qt);
  int q0 = t.q0, q1 = t.q0 + t.rows - 1;
  ks.base = 0; ks.kend = g.S;
  // touching range [lo, hi] and fully-inside range [fi, fl] (may be empty)
  int lo = imax(0, q0 - g.hw) / kTile;
  int hi = imin(g.S - 1, q1 + g.hw) / kTile;
  if (seg == 0) {
    ks.r0b = lo; ks.r0e = hi + 1; ks.r1b = ks.r1e = 0;
    return ks;
  }
  int fi = lo, fl = hi;
  while (fi <= fl && !wtile_inside(g, q0, q1, fi)) ++fi;
  while (fl >= fi && !wtile_inside(g, q0, q1, fl)) --fl;
  if (fi > fl) {            // no tile fully inside: complement spans everything
    ks.r0b = 0; ks.r0e = g.nkt; ks.r1b = ks.r1e = 0;
  } else {
    ks.r0b = 0; ks.r0e = fi; ks.r1b = fl + 1; ks.r1e = g.nkt;
  }
  return ks;
}

// Distinct 128x128 blocks of key set `seg` of query tile `qt` that count as
// "computed" (or "skipped") blocks: in window mode the straddling tiles are
// counted once, in the window set.
template <int W = -1>
DT_HD int counted_blocks(const Geom& g, int qt, int seg) {
  KeySet ks = key_set<W>(g, qt, seg);
  if (!is_window<W>(g) || seg == 0) return ks.ntiles();
  QTile t = query_tile<W>(g, qt);
  int q0 = t.q0, q1 = t.q0 + t.rows - 1, n = 0;
  for (int i = 0; i < ks.ntiles(); ++i)
    if (!wtile_touches(g, q0, q1, ks.tile(i))) ++n;
  return n;
}

}  // namespace dt
