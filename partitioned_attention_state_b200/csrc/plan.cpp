// plan.cpp -- host-side plan builder of libdt (integer work only).
//
// "DiTango: Cost-Effective Parallel Diffusion Generation with Selective
// Attention State Reuse": selective compute and reuse (Fig. 6) -- each query
// partition computes its own and nearby partitions and reuses cached states of
// distant ones; spatial locality (Fig. 5a) ranks partitions by distance; anchor
// steps compute everything.  "DiTFastAttn: Attention Compression for Diffusion
// Transformer Models" (Approach): window attention with a cached residual is
// expressed as two key sets per query tile (window, complement).  State
// grouping (grouping of spatially adjacent states) makes a key set a group of
// partitions; the proximity rule then ranks groups.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <vector>

#include "../../include/dt.h"
#include "geometry.h"

namespace {

bool params_ok(const dt_plan_params* p) {
  if (!p) return false;
  if (p->H < 0 || p->S < 0 || p->D < 1 || p->step < 1) return false;
  if (p->mode < DT_MODE_ALL_COMPUTE || p->mode > DT_MODE_ANCHOR) return false;
  if (p->group < 0) return false;
  if (p->mode == DT_MODE_WINDOW) {
    if (p->window < 1 || p->group != 0) return false;
  } else {
    if (p->P < 1) return false;
    const int rmax = p->group > 0 ? dt::ceil_div(p->P, p->group) : p->P - 1;
    if ((p->mode == DT_MODE_PROXIMITY || p->mode == DT_MODE_IMPORTANCE) &&
        (p->reuse_per_row < 0 || p->reuse_per_row > rmax))
      return false;
  }
  return true;
}

dt::Geom geom_of(const dt_plan_params* p) {
  return p->mode == DT_MODE_WINDOW ? dt::make_geom(p->H, p->S, p->D, 1, p->window)
                                   : dt::make_geom(p->H, p->S, p->D, p->P, 0, p->group);
}

// Grouped proximity row of a query in partition q (1 + m entries): set 0 (the
// local partition) is computed; the r groups farthest from q's group are
// reused, equal distances in increasing index order.
void group_proximity_row(int q, int m, int g, int r, uint8_t* row) {
  for (int k = 0; k <= m; ++k) row[k] = DT_PLAN_COMPUTE;
  const int lg = q / g;
  int taken = 0;
  for (int dist = m - 1; dist >= 0 && taken < r; --dist) {
    int cand[2] = {lg - dist, lg + dist};
    for (int c = 0; c < (dist == 0 ? 1 : 2) && taken < r; ++c) {
      if (cand[c] >= 0 && cand[c] < m) { row[1 + cand[c]] = DT_PLAN_REUSE; ++taken; }
    }
  }
}

// Keys of key set k of query tile qt (partition modes).
int64_t set_keys(const dt::Geom& g, int qt, int k) {
  if (g.grp == 0) return dt::part_end(g, k) - dt::part_begin(g, k);
  const int q = dt::query_tile<0>(g, qt).part;
  if (k == 0) return dt::part_end(g, q) - dt::part_begin(g, q);
  const int a = (k - 1) * g.grp, b = dt::imin(k * g.grp, g.parts);
  int64_t n = dt::part_end(g, b - 1) - dt::part_begin(g, a);
  if (a <= q && q < b) n -= dt::part_end(g, q) - dt::part_begin(g, q);
  return n;
}

// Proximity row of query partition q: reuse the r partitions farthest from q,
// equal distances in increasing index order; q itself is never reused.
void proximity_row(int q, int P, int r, uint8_t* row) {
  for (int k = 0; k < P; ++k) row[k] = DT_PLAN_COMPUTE;
  int taken = 0;
  for (int dist = P - 1; dist >= 1 && taken < r; --dist) {
    int cand[2] = {q - dist, q + dist};
    for (int c = 0; c < 2 && taken < r; ++c) {
      if (cand[c] >= 0 && cand[c] < P) { row[cand[c]] = DT_PLAN_REUSE; ++taken; }
    }
  }
}

int64_t window_pairs(const dt::Geom& g, int q0, int rows) {
  int64_t n = 0;
  for (int i = q0; i < q0 + rows; ++i)
    n += dt::imin(g.S - 1, i + g.hw) - dt::imax(0, i - g.hw) + 1;
  return n;
}

}  // namespace

extern "C" const char* dt_status_string(int s) {
  switch (s) {
    case DT_OK: return "DT_OK";
    case DT_ERR_INVALID: return "DT_ERR_INVALID: invalid argument";
    case DT_ERR_UNSUPPORTED: return "DT_ERR_UNSUPPORTED: unsupported head dim or misaligned pointer";
    case DT_ERR_CACHE_EMPTY: return "DT_ERR_CACHE_EMPTY: reuse of a cache slot never written";
    case DT_ERR_CUDA: return "DT_ERR_CUDA: CUDA call failed";
    case DT_ERR_TIMEOUT: return "DT_ERR_TIMEOUT: a bounded device wait ran out";
    default: return "unknown dt status";
  }
}

extern "C" int dt_key_set_tiles(const dt_plan_params* p, int32_t qt, int32_t k, int32_t* row0, int32_t* rowend,
                                int32_t cap) {
  if (!params_ok(p) || cap < 0 || (cap > 0 && (!row0 || !rowend))) return DT_ERR_INVALID;
  dt::Geom g = geom_of(p);
  if (qt < 0 || qt >= g.nqt || k < 0 || k >= g.P) return DT_ERR_INVALID;
  const dt::KeySet ks = dt::key_set(g, qt, k);
  const int nt = ks.ntiles();
  for (int i = 0; i < nt && i < cap; ++i) {
    const int t = ks.tile(i);
    row0[i] = ks.row0(t);
    rowend[i] = ks.rowend(t);
  }
  return nt;
}

extern "C" int dt_plan_geometry(const dt_plan_params* p, int32_t* nqt, int32_t* nseg) {
  if (!params_ok(p) || !nqt || !nseg) return DT_ERR_INVALID;
  dt::Geom g = geom_of(p);
  *nqt = g.nqt;
  *nseg = g.P;
  return DT_OK;
}

namespace {
int finish_plan(const dt_plan_params* p, const dt::Geom& g, dt_plan* out);
}

extern "C" int dt_plan_build(const dt_plan_params* p, const uint8_t* explicit_plan, dt_plan* out) {
  if (!params_ok(p) || !out || !out->plan) return DT_ERR_INVALID;
  if (p->mode == DT_MODE_IMPORTANCE || p->mode == DT_MODE_ANCHOR) return DT_ERR_INVALID;   // needs their state
  dt::Geom g = geom_of(p);
  const int nqt = g.nqt, nseg = g.P;
  out->nqt = nqt;
  out->nseg = nseg;
  out->computed_blocks = out->skipped_blocks = out->computed_flops = 0;
  const bool anchor = p->step <= 1;
  uint8_t* plan = out->plan;

  for (int qt = 0; qt < nqt; ++qt) {
    uint8_t* row = plan + (size_t)qt * nseg;
    switch (p->mode) {
      case DT_MODE_ALL_COMPUTE:
        for (int k = 0; k < nseg; ++k) row[k] = DT_PLAN_COMPUTE;
        break;
      case DT_MODE_PROXIMITY:
        if (anchor) { for (int k = 0; k < nseg; ++k) row[k] = DT_PLAN_COMPUTE; }
        else if (g.grp > 0) group_proximity_row(dt::query_tile(g, qt).part, nseg - 1, g.grp, p->reuse_per_row, row);
        else proximity_row(dt::query_tile(g, qt).part, nseg, p->reuse_per_row, row);
        break;
      case DT_MODE_ALL_REUSE:
        for (int k = 0; k < nseg; ++k) row[k] = DT_PLAN_REUSE;
        break;
      case DT_MODE_EXPLICIT:
        if (!explicit_plan) return DT_ERR_INVALID;
        for (int k = 0; k < nseg; ++k) {
          uint8_t v = explicit_plan[(size_t)qt * nseg + k];
          if (v != DT_PLAN_COMPUTE && v != DT_PLAN_REUSE) return DT_ERR_INVALID;
          row[k] = v;
        }
        break;
      case DT_MODE_WINDOW:
        row[0] = DT_PLAN_COMPUTE;
        row[1] = anchor ? DT_PLAN_COMPUTE : DT_PLAN_REUSE;
        break;
    }
  }
  return finish_plan(p, g, out);
}

extern "C" int dt_plan_build_importance(const dt_plan_params* p, const float* weights, dt_plan* out) {
  if (!params_ok(p) || !out || !out->plan || p->mode != DT_MODE_IMPORTANCE) return DT_ERR_INVALID;
  dt::Geom g = geom_of(p);
  const int nqt = g.nqt, nseg = g.P;
  if (!weights && p->step > 1 && nqt > 0) return DT_ERR_INVALID;
  out->nqt = nqt;
  out->nseg = nseg;
  out->computed_blocks = out->skipped_blocks = out->computed_flops = 0;
  for (int qt = 0; qt < nqt; ++qt) {
    uint8_t* row = out->plan + (size_t)qt * nseg;
    for (int k = 0; k < nseg; ++k) row[k] = DT_PLAN_COMPUTE;
    if (p->step <= 1) continue;                                   // anchor
    const int local = g.grp > 0 ? 0 : dt::query_tile<0>(g, qt).part;
    const float* w = weights + (size_t)qt * nseg;
    const int32_t* st = out->stamps ? out->stamps + (size_t)qt * nseg : nullptr;
    // r times: the eligible set of smallest predicted error, lower index on ties
    for (int taken = 0; taken < p->reuse_per_row; ++taken) {
      int best = -1;
      float best_e = 0.f;
      for (int k = 0; k < nseg; ++k) {
        if (k == local || row[k] == DT_PLAN_REUSE || !st || st[k] < 0) continue;
        const float e = w[k] * (float)(p->step - st[k]);
        if (best < 0 || e < best_e) { best = k; best_e = e; }
      }
      if (best < 0) break;
      row[best] = DT_PLAN_REUSE;
    }
  }
  return finish_plan(p, g, out);
}


extern "C" int dt_plan_share_counts(const dt_plan_params* p, int32_t kind, dt_plan* io) {
  if (!params_ok(p) || !io) return DT_ERR_INVALID;
  if (kind == DT_SHARE_CFG) {
    // the plan's counts are H x (per-head counts), so halving is exact
    if (p->H % 2 != 0) return DT_ERR_INVALID;
    const int64_t total = io->computed_blocks + io->skipped_blocks;
    io->computed_blocks /= 2;
    io->skipped_blocks = total - io->computed_blocks;
    io->computed_flops /= 2;
    return DT_OK;
  }
  if (kind != DT_SHARE_TIMESTEP) return DT_ERR_INVALID;
  const dt::Geom g = geom_of(p);
  int64_t total = 0;
  for (int qt = 0; qt < g.nqt; ++qt)
    for (int k = 0; k < g.P; ++k) total += (int64_t)p->H * dt::counted_blocks(g, qt, k);
  io->computed_blocks = 0;
  io->skipped_blocks = total;
  io->computed_flops = 0;
  return DT_OK;
}

namespace {

// The local key set of query tile qt: its own partition, or set 0 with grouping.
int local_set(const dt::Geom& g, int qt) { return g.grp > 0 ? 0 : dt::query_tile<0>(g, qt).part; }

bool anchor_state_ok(const dt_plan_params* p, const dt_anchor_state* a) {
  return params_ok(p) && a && p->mode == DT_MODE_ANCHOR && a->weights && a->alpha && a->drift;
}

}  // namespace

extern "C" int dt_anchor_init(const dt_plan_params* p, dt_anchor_state* a) {
  if (!anchor_state_ok(p, a)) return DT_ERR_INVALID;
  const dt::Geom g = geom_of(p);
  const size_t n = (size_t)g.nqt * g.P;
  for (size_t i = 0; i < n; ++i) { a->weights[i] = 0.f; a->alpha[i] = 1.f; }
  for (int t = 0; t < g.nqt; ++t) a->drift[t] = 0.f;
  a->eps = 0.f;
  a->last_anchor = 0;
  a->anchored = 0;
  return DT_OK;
}

extern "C" int dt_plan_build_anchor(const dt_plan_params* p, dt_anchor_state* a, dt_plan* out) {
  if (!anchor_state_ok(p, a) || !out || !out->plan) return DT_ERR_INVALID;
  const dt::Geom g = geom_of(p);
  const int nqt = g.nqt, nseg = g.P;
  out->nqt = nqt;
  out->nseg = nseg;
  out->computed_blocks = out->skipped_blocks = out->computed_flops = 0;
  bool anchor = p->step <= 1;
  for (int t = 0; t < nqt && !anchor; ++t) anchor = a->drift[t] > a->theta;
  a->anchored = anchor ? 1 : 0;
  for (int qt = 0; qt < nqt; ++qt) {
    uint8_t* row = out->plan + (size_t)qt * nseg;
    for (int k = 0; k < nseg; ++k) row[k] = DT_PLAN_COMPUTE;
    if (anchor) continue;
    const int loc = local_set(g, qt);
    const int32_t* st = out->stamps ? out->stamps + (size_t)qt * nseg : nullptr;
    for (int k = 0; k < nseg; ++k) {
      if (k == loc || !st || st[k] < 0) continue;
      const float ase = (a->weights[(size_t)qt * nseg + k] * a->alpha[(size_t)qt * nseg + k]) * (float)(p->step - st[k]);
      if (ase <= a->eps) row[k] = DT_PLAN_REUSE;
    }
  }
  return finish_plan(p, g, out);
}

extern "C" int dt_anchor_update(const dt_plan_params* p, dt_anchor_state* a, const int32_t* stamps_before,
                                const uint8_t* plan, const float* err, const float* weights_now) {
  if (!anchor_state_ok(p, a) || !stamps_before || !plan || !err) return DT_ERR_INVALID;
  if (a->anchored && !weights_now) return DT_ERR_INVALID;
  const dt::Geom g = geom_of(p);
  const int nqt = g.nqt, nseg = g.P, H = p->H;
  // error of pair (qt, k): sums over heads and the 4 row groups in increasing
  // order, in double; false if the pair has no previous state or was not computed
  auto pair_error = [&](int qt, int k, float* e) -> bool {
    const size_t i = (size_t)qt * nseg + k;
    if (plan[i] != DT_PLAN_COMPUTE || stamps_before[i] < 0) return false;
    double diff = 0.0, norm = 0.0;
    for (int h = 0; h < H; ++h)
      for (int w = 0; w < 4; ++w) {
        const float* e2 = err + (((i * H) + h) * 4 + w) * 2;
        diff += (double)e2[0];
        norm += (double)e2[1];
      }
    *e = norm > 0.0 ? (float)std::sqrt(diff / norm) : 0.f;
    return true;
  };
  if (!a->anchored) {
    for (int qt = 0; qt < nqt; ++qt) {
      float e;
      if (pair_error(qt, local_set(g, qt), &e)) a->drift[qt] = a->drift[qt] + e;
    }
    return DT_OK;
  }
  a->last_anchor = p->step;
  std::vector<float> rates;
  rates.reserve((size_t)nqt * nseg);
  for (int qt = 0; qt < nqt; ++qt) {
    a->drift[qt] = 0.f;
    const int loc = local_set(g, qt);
    for (int k = 0; k < nseg; ++k) {
      const size_t i = (size_t)qt * nseg + k;
      a->weights[i] = weights_now[i];
      if (k == loc) continue;
      float e;
      if (pair_error(qt, k, &e)) a->alpha[i] = e / (float)(p->step - stamps_before[i]);
      rates.push_back(a->weights[i] * a->alpha[i]);
    }
  }
  std::sort(rates.begin(), rates.end());
  const int64_t n = rates.empty() ? 0 : (int64_t)std::ceil((double)a->target_ratio * (double)rates.size() - 1e-9);
  a->eps = n > 0 ? rates[(size_t)std::min<int64_t>(n, (int64_t)rates.size()) - 1] : 0.f;
  return DT_OK;
}

namespace {

// Shared tail of the plan builders: refuse REUSE of never-written slots,
// stamp the COMPUTE slots, fill the counts.
int finish_plan(const dt_plan_params* p, const dt::Geom& g, dt_plan* out) {
  const int nqt = g.nqt, nseg = g.P;
  uint8_t* plan = out->plan;
  // validate reuse against stamps before touching them
  const size_t n = (size_t)nqt * nseg;
  for (size_t i = 0; i < n; ++i) {
    if (plan[i] == DT_PLAN_REUSE) {
      int32_t s = out->stamps ? out->stamps[i] : -1;
      if (s < 0) return DT_ERR_CACHE_EMPTY;
    }
  }
  if (out->stamps)
    for (size_t i = 0; i < n; ++i)
      if (plan[i] == DT_PLAN_COMPUTE) out->stamps[i] = p->step;

  // counts
  int64_t cb = 0, sb = 0, fl = 0;
  const int64_t H = p->H, D = p->D;
  for (int qt = 0; qt < nqt; ++qt) {
    const uint8_t* row = plan + (size_t)qt * nseg;
    dt::QTile t = dt::query_tile(g, qt);
    if (p->mode == DT_MODE_WINDOW) {
      int band = dt::counted_blocks(g, qt, 0);
      int outside = dt::counted_blocks(g, qt, 1);
      if (row[1] == DT_PLAN_COMPUTE) {
        cb += H * (band + outside);
        fl += 4 * H * D * (int64_t)t.rows * g.S;
      } else {
        cb += H * band;
        sb += H * outside;
        fl += 4 * H * D * window_pairs(g, t.q0, t.rows);
      }
    } else {
      for (int k = 0; k < nseg; ++k) {
        const int64_t len = set_keys(g, qt, k);
        int64_t nb = H * dt::counted_blocks(g, qt, k);
        if (row[k] == DT_PLAN_COMPUTE) {
          cb += nb;
          fl += 4 * H * D * (int64_t)t.rows * len;
        } else {
          sb += nb;
        }
      }
    }
  }
  out->computed_blocks = cb;
  out->skipped_blocks = sb;
  out->computed_flops = fl;
  return DT_OK;
}

}  // namespace
