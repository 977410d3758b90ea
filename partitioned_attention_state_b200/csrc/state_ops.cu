// state_ops.cu -- HBM-bound state kernels of libdt: N-way state composition,
// plan-driven cache scatter, in-place regrouping of cached group states,
// partition importance, and the window residual (make / apply).
//
// All three stream rows of D fp32 values with 16-byte vector accesses over a
// flat index, so consecutive threads touch consecutive 16-byte words (fully
// coalesced); grids are sized in multiples of the SM count.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "../../include/dt.h"
#include "geometry.h"
#include "state_ops.h"

namespace dt {
namespace {

constexpr int kBlock = 256;
__device__ __forceinline__ float neg_inf() { return -__int_as_float(0x7f800000); }
#define kNegInf (neg_inf())

// "DiTango", composition of attention states (Eq. 4), N-way: per row one max
// over the N log-sum-exps, then weights e^(L_n - L).
__global__ void __launch_bounds__(kBlock) state_merge_kernel(int N, int64_t rows, int D, int64_t plane,
                                                             const float* __restrict__ O_in,
                                                             const float* __restrict__ L_in,
                                                             float* __restrict__ O_out, float* __restrict__ L_out) {
  const int d4n = D / 4;
  const int64_t total = rows * d4n;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / d4n;
    const int c4 = (int)(i - row * d4n);
    float M = kNegInf;
    for (int n = 0; n < N; ++n) M = fmaxf(M, __ldg(L_in + n * rows + row));
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float Lr = kNegInf;
    if (M > kNegInf) {
      float tot = 0.f;
      for (int n = 0; n < N; ++n) tot += expf(__ldg(L_in + n * rows + row) - M);
      Lr = M + logf(tot);
      for (int n = 0; n < N; ++n) {
        const float w = expf(__ldg(L_in + n * rows + row) - Lr);
        const float4 v = __ldg(reinterpret_cast<const float4*>(O_in + n * plane + row * D) + c4);
        acc.x = fmaf(w, v.x, acc.x);
        acc.y = fmaf(w, v.y, acc.y);
        acc.z = fmaf(w, v.z, acc.z);
        acc.w = fmaf(w, v.w, acc.w);
      }
    }
    reinterpret_cast<float4*>(O_out + row * D)[c4] = acc;
    if (c4 == 0) L_out[row] = Lr;
  }
}

// "DiTango": freshly computed states are stored in the attention state cache;
// a slot is written iff its (query tile, partition) entry is COMPUTE.
__global__ void __launch_bounds__(kBlock) cache_update_kernel(Geom G, const uint8_t* __restrict__ plan,
                                                              const float* __restrict__ fO,
                                                              const float* __restrict__ fL, float* __restrict__ cO,
                                                              float* __restrict__ cL) {
  const int d4n = G.D / 4;
  const int64_t rows = (int64_t)G.P * G.H * G.S;
  const int64_t total = rows * d4n;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / d4n;              // ((k * H + h) * S + s)
    const int c4 = (int)(i - row * d4n);
    const int s = (int)(row % G.S);
    const int k = (int)(row / ((int64_t)G.H * G.S));
    const int part = s / G.c;
    const int qt = part * G.tpp + (s - part_begin(G, part)) / kTile;
    if (plan[(size_t)qt * G.P + k] != DT_PLAN_COMPUTE) continue;
    reinterpret_cast<float4*>(cO + row * G.D)[c4] = __ldg(reinterpret_cast<const float4*>(fO + row * G.D) + c4);
    if (c4 == 0) cL[row] = __ldg(fL + row);
  }
}

// "DiTFastAttn", window attention with residual sharing.
__global__ void __launch_bounds__(kBlock) window_residual_kernel(int op, int64_t n4, const float* __restrict__ Of,
                                                                 const float* __restrict__ Ow, float* __restrict__ R,
                                                                 __nv_bfloat16* __restrict__ O) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
    const float4 w = __ldg(reinterpret_cast<const float4*>(Ow) + i);
    if (op == DT_WR_MAKE) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(Of) + i);
      reinterpret_cast<float4*>(R)[i] = make_float4(f.x - w.x, f.y - w.y, f.z - w.z, f.w - w.w);
    } else {
      const float4 r = __ldg(reinterpret_cast<const float4*>(R) + i);
      __nv_bfloat162 lo = __floats2bfloat162_rn(w.x + r.x, w.y + r.y);
      __nv_bfloat162 hi = __floats2bfloat162_rn(w.z + r.z, w.w + r.w);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t*>(&lo);
      pk.y = *reinterpret_cast<uint32_t*>(&hi);
      reinterpret_cast<uint2*>(O)[i] = pk;
    }
  }
}

// "DiTango", Dynamic Group State Compose: cached group states are merged
// `factor` at a time into coarser groups (Eq. 4 composition), in place.  One
// warp owns a (head, row) and walks the new groups in increasing order; new
// group i reads old slots 1 + factor*i .. (all at or after slot 1 + i) and
// writes slot 1 + i, which only an already finished group read.  Inside a
// group every lane reads all inputs (the LSEs are shared by the whole row)
// before any lane writes, so the write of slot 1 + i cannot race a read of it.
// F (>= factor) bounds the inputs a lane loads at once.
template <int F>
__global__ void __launch_bounds__(kBlock) group_compose_kernel(int m, int factor, int64_t rows, int D,
                                                               float* __restrict__ cO, float* __restrict__ cL) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (kBlock / 32);
  const int m2 = (m + factor - 1) / factor;
  const int d4n = D / 4;
  for (int64_t row = blockIdx.x * (int64_t)(kBlock / 32) + (threadIdx.x >> 5); row < rows; row += warps) {
    for (int i = 0; i < m2; ++i) {
      const int j0 = 1 + factor * i, n = min(factor, m - factor * i);
      // all reads of this group first, issued together: the LSEs and this
      // lane's OUT columns (a slot with LSE -inf gets weight 0 and its OUT,
      // possibly never written, is replaced by zeros after the load)
      float lv[F];
      float4 v[F];
      const bool one = d4n <= 32;               // D <= 128: one float4 per lane
#pragma unroll
      for (int k = 0; k < F; ++k) {
        lv[k] = k < n ? cL[(int64_t)(j0 + k) * rows + row] : kNegInf;
        v[k] = (one && k < n && lane < d4n)
                   ? reinterpret_cast<const float4*>(cO + ((int64_t)(j0 + k) * rows + row) * D)[lane]
                   : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      float M = lv[0];
#pragma unroll
      for (int k = 1; k < F; ++k) M = fmaxf(M, lv[k]);
      float w[F];
      float Lr = kNegInf;
      if (M > kNegInf) {
        float tot = 0.f;
#pragma unroll
        for (int k = 0; k < F; ++k) tot += k < n ? expf(lv[k] - M) : 0.f;
        Lr = M + logf(tot);
      }
#pragma unroll
      for (int k = 0; k < F; ++k) w[k] = (k < n && lv[k] > kNegInf) ? expf(lv[k] - Lr) : 0.f;
      for (int c4 = lane; c4 < d4n; c4 += 32) {
        if (!one) {
#pragma unroll
          for (int k = 0; k < F; ++k)
            v[k] = k < n ? reinterpret_cast<const float4*>(cO + ((int64_t)(j0 + k) * rows + row) * D)[c4]
                         : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int k = 0; k < F; ++k)
          if (w[k] == 0.f) v[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < F; ++k) {
          acc.x = fmaf(w[k], v[k].x, acc.x);
          acc.y = fmaf(w[k], v[k].y, acc.y);
          acc.z = fmaf(w[k], v[k].z, acc.z);
          acc.w = fmaf(w[k], v[k].w, acc.w);
        }
        __stcs(reinterpret_cast<float4*>(cO + ((int64_t)(1 + i) * rows + row) * D) + c4, acc);
      }
      __syncwarp();                             // every lane has read this group's LSEs
      if (lane == 0) cL[(int64_t)(1 + i) * rows + row] = Lr;
      __syncwarp();
    }
  }
}

// The same regrouping with every input of a row held at once (m <= MAXM old
// groups, D <= 128 so that a lane owns one float4 of a row): all loads of the
// row are issued before any store, so a row costs one memory round trip
// instead of one per new group.  The warp synchronises once between its loads
// and its stores, after which no old value of the row is read again.
template <int MAXM>
__global__ void __launch_bounds__(kBlock) group_compose_row_kernel(int m, int factor, int64_t rows, int D,
                                                                   float* __restrict__ cO, float* __restrict__ cL) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (kBlock / 32);
  const int m2 = (m + factor - 1) / factor;
  const bool on = lane < D / 4;
  for (int64_t row = blockIdx.x * (int64_t)(kBlock / 32) + (threadIdx.x >> 5); row < rows; row += warps) {
    float lv[MAXM];
    float4 v[MAXM];
#pragma unroll
    for (int k = 0; k < MAXM; ++k) {
      lv[k] = k < m ? cL[(int64_t)(1 + k) * rows + row] : kNegInf;
      v[k] = (k < m && on) ? __ldcs(reinterpret_cast<const float4*>(cO + ((int64_t)(1 + k) * rows + row) * D) + lane)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncwarp();
    for (int i = 0; i < m2; ++i) {
      const int j0 = factor * i, j1 = min(j0 + factor, m);
      float M = kNegInf;
#pragma unroll
      for (int k = 0; k < MAXM; ++k)
        if (k >= j0 && k < j1) M = fmaxf(M, lv[k]);
      float Lr = kNegInf;
      if (M > kNegInf) {
        float tot = 0.f;
#pragma unroll
        for (int k = 0; k < MAXM; ++k)
          if (k >= j0 && k < j1) tot += expf(lv[k] - M);
        Lr = M + logf(tot);
      }
      // a slot with LSE -inf (possibly never written) gets weight 0 and is not read
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < MAXM; ++k) {
        const float wk = (k >= j0 && k < j1 && lv[k] > kNegInf) ? expf(lv[k] - Lr) : 0.f;
        if (wk != 0.f) {
          acc.x = fmaf(wk, v[k].x, acc.x);
          acc.y = fmaf(wk, v[k].y, acc.y);
          acc.z = fmaf(wk, v[k].z, acc.z);
          acc.w = fmaf(wk, v[k].w, acc.w);
        }
      }
      if (on) __stcs(reinterpret_cast<float4*>(cO + ((int64_t)(1 + i) * rows + row) * D) + lane, acc);
      if (lane == 0) cL[(int64_t)(1 + i) * rows + row] = Lr;
    }
  }
}

// "DiTango", partition importance: the normalised composition weight
// exp(LSE_k - LSE) of key set k for each row, averaged over the rows of a
// query tile and the heads.  One block per (query tile, key set).
constexpr int kImpBlock = 128;   // one thread per row of a query tile
__global__ void __launch_bounds__(kImpBlock) state_importance_kernel(Geom G, const float* __restrict__ cL,
                                                                     const float* __restrict__ L,
                                                                     float* __restrict__ w) {
  __shared__ float part[kImpBlock / 32];
  const int qt = blockIdx.x / G.P, k = blockIdx.x - qt * G.P;
  const QTile t = query_tile<kModePartition>(G, qt);
  const int n = G.H * t.rows;
  float acc = 0.f;
  if ((int)threadIdx.x < t.rows) {
    // thread t owns row q0 + t and walks the heads with 8 loads of each array
    // in flight; a warp's loads cover 32 consecutive rows (128 bytes)
    const int r = t.q0 + threadIdx.x;
    const float* lk = cL + (int64_t)k * G.H * G.S + r;
    const float* lt = L + r;
    int h = 0;
    for (; h + 8 <= G.H; h += 8) {
      float a[8], b[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        a[u] = __ldcs(lk + (int64_t)(h + u) * G.S);
        b[u] = lt[(int64_t)(h + u) * G.S];
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (a[u] > kNegInf && b[u] > kNegInf) acc += expf(a[u] - b[u]);
    }
    for (; h < G.H; ++h) {
      const float a = __ldcs(lk + (int64_t)h * G.S), b = lt[(int64_t)h * G.S];
      if (a > kNegInf && b > kNegInf) acc += expf(a - b);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
    for (int j = 0; j < kImpBlock / 32; ++j) tot += part[j];
    w[blockIdx.x] = n > 0 ? tot / (float)n : 0.f;
  }
}

// "DiTFastAttn", attention sharing across CFG branches: the unconditional
// branch takes the conditional branch's attention, so the states the
// conditional heads computed this step also become the unconditional heads'
// cached states.  For every (query tile, key set) the plan marks COMPUTE,
// the slot rows of head h < hb are copied to head h + hb (cache_O as fp32 or
// bf16, cache_L fp32); in window mode a computed complement copies the rows
// of R instead.  One thread per 16-byte vector.
__global__ void __launch_bounds__(kBlock) share_states_kernel(Geom G, const uint8_t* __restrict__ plan, int hb,
                                                              int elem_bytes, uint8_t* __restrict__ cO,
                                                              float* __restrict__ cL, float* __restrict__ R) {
  const bool win = G.window > 0;
  const int vec = 16 / elem_bytes;                       // elements per 16-byte vector
  const int dv = G.D / vec;
  const int nk = win ? 1 : G.P;
  const int64_t rows = (int64_t)nk * hb * G.S;
  const int64_t total = rows * dv;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / dv;                          // ((k * hb + h) * S + s)
    const int c = (int)(i - row * dv);
    const int s = (int)(row % G.S);
    const int h = (int)((row / G.S) % hb);
    const int k = (int)(row / ((int64_t)hb * G.S));
    int qt;
    if (win) {
      qt = s / kTile;
    } else {
      const int part = s / G.c;
      qt = part * G.tpp + (s - part_begin(G, part)) / kTile;
    }
    const int seg = win ? 1 : k;
    if ((plan[(size_t)qt * G.P + seg] & 1u) == 0) continue;
    if (win) {
      const float4* src = reinterpret_cast<const float4*>(R + ((int64_t)h * G.S + s) * G.D);
      float4* dst = reinterpret_cast<float4*>(R + ((int64_t)(h + hb) * G.S + s) * G.D);
      dst[c] = src[c];
    } else {
      const int64_t from = ((int64_t)k * G.H + h) * G.S + s, to = ((int64_t)k * G.H + h + hb) * G.S + s;
      reinterpret_cast<uint4*>(cO + to * G.D * elem_bytes)[c] =
          reinterpret_cast<const uint4*>(cO + from * G.D * elem_bytes)[c];
      if (c == 0) cL[to] = cL[from];
    }
  }
}

__global__ void __launch_bounds__(kBlock) fill_zero_kernel(float* __restrict__ x, int64_t n) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    x[i] = 0.f;
}

int grid_for(int64_t work, int sms) {
  int64_t blocks = (work + kBlock - 1) / kBlock;
  int64_t cap = (int64_t)sms * 8;           // 8 resident 256-thread blocks per SM
  if (blocks > cap) blocks = cap;
  return blocks < 1 ? 1 : (int)blocks;
}

}  // namespace

int launch_state_merge(int N, int H, int S, int D, const float* O_in, const float* L_in, float* O_out,
                       float* L_out, int sms, cudaStream_t st) {
  const int64_t rows = (int64_t)H * S;
  state_merge_kernel<<<grid_for(rows * (D / 4), sms), kBlock, 0, st>>>(N, rows, D, rows * D, O_in, L_in, O_out,
                                                                       L_out);
  return cudaGetLastError() == cudaSuccess ? DT_OK : DT_ERR_CUDA;
}

int launch_cache_update(const Geom& G, const uint8_t* plan, const float* fO, const float* fL, float* cO, float* cL,
                        int sms, cudaStream_t st) {
  const int64_t work = (int64_t)G.P * G.H * G.S * (G.D / 4);
  cache_update_kernel<<<grid_for(work, sms), kBlock, 0, st>>>(G, plan, fO, fL, cO, cL);
  return cudaGetLastError() == cudaSuccess ? DT_OK : DT_ERR_CUDA;
}

int launch_group_compose(int m, int factor, int H, int S, int D, float* cO, float* cL, int sms, cudaStream_t st) {
  const int64_t rows = (int64_t)H * S;
  const int grid = grid_for(rows * 32, sms);
  if (D <= 128 && m <= 16) {   // every input of a row at once
    if (m <= 4) group_compose_row_kernel<4><<<grid, kBlock, 0, st>>>(m, factor, rows, D, cO, cL);
    else if (m <= 8) group_compose_row_kernel<8><<<grid, kBlock, 0, st>>>(m, factor, rows, D, cO, cL);
    else group_compose_row_kernel<16><<<grid, kBlock, 0, st>>>(m, factor, rows, D, cO, cL);
    return cudaGetLastError() == cudaSuccess ? DT_OK : DT_ERR_CUDA;
  }
  switch (factor) {   // the factor bounds how many inputs a lane loads at once
    case 2: group_compose_kernel<2><<<grid, kBlock, 0, st>>>(m, factor, rows, D, cO, cL); break;
    case 3: group_compose_kernel<3><<<grid, kBlock, 0, st>>>(m, factor, rows, D, cO, cL); break;
    case 4: group_compose_kernel<4><<<grid, kBlock, 0, st>>>(m, factor, rows, D, cO, cL); break;
    default: group_compose_kernel<8><<<grid, kBlock, 0, st>>>(m, factor, rows, D, cO, cL); break;   // 5..8
  }
  return cudaGetLastError() == cudaSuccess ? DT_OK : DT_ERR_CUDA;
}

int launch_state_importance(const Geom& G, const float* cL, const float* L, float* w, cudaStream_t st) {
  const int64_t blocks = (int64_t)G.nqt * G.P;
  state_importance_kernel<<<(unsigned)blocks, kImpBlock, 0, st>>>(G, cL, L, w);
  return cudaGetLastError() == cudaSuccess ? DT_OK : DT_ERR_CUDA;
}

int launch_share_states(const Geom& G, const uint8_t* plan, int hb, int elem_bytes, void* cO, float* cL, float* R,
                        int sms, cudaStream_t st) {
  const int nk = G.window > 0 ? 1 : G.P;
  const int64_t work = (int64_t)nk * hb * G.S * (G.D * elem_bytes / 16);
  if (work == 0) return DT_OK;
  share_states_kernel<<<grid_for(work, sms), kBlock, 0, st>>>(G, plan, hb, elem_bytes,
                                                              reinterpret_cast<uint8_t*>(cO), cL, R);
  return cudaGetLastError() == cudaSuccess ? DT_OK : DT_ERR_CUDA;
}

int launch_fill_zero(float* x, int64_t n, cudaStream_t st) {
  fill_zero_kernel<<<(unsigned)((n + kBlock - 1) / kBlock < 1024 ? (n + kBlock - 1) / kBlock : 1024), kBlock, 0, st>>>(x, n);
  return cudaGetLastError() == cudaSuccess ? DT_OK : DT_ERR_CUDA;
}

int launch_window_residual(int op, int64_t n, const float* Of, const float* Ow, float* R, void* O, int sms,
                           cudaStream_t st) {
  const int64_t n4 = n / 4;
  window_residual_kernel<<<grid_for(n4, sms), kBlock, 0, st>>>(op, n4, Of, Ow, R,
                                                              reinterpret_cast<__nv_bfloat16*>(O));
  return cudaGetLastError() == cudaSuccess ? DT_OK : DT_ERR_CUDA;
}

}  // namespace dt
