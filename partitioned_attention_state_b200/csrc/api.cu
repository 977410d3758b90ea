// api.cu -- extern "C" device entry points of libdt: argument validation,
// TMA descriptor encoding and kernel launches.  No allocation happens here.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>
#include <cstring>

#include "../../include/dt.h"
#include "attn_fused.h"
#include "geometry.h"
#include "state_ops.h"

namespace {

std::atomic<long long> g_wait_limit_ns{2000000000ll};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count(int* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DT_ERR_CUDA;
  static int cached[64] = {0};
  if (dev >= 0 && dev < 64 && cached[dev] > 0) { *out = cached[dev]; return DT_OK; }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return DT_ERR_CUDA;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  *out = n;
  return DT_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// bf16 [H][S][D] viewed as a 3-D tensor (D, S, H); box (bw, 128, 1).
bool encode_qkv(CUtensorMap* m, const void* base, int H, int S, int D, int bw, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)S, (cuuint64_t)H};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)S * D * 2};
  cuuint32_t box[3] = {(cuuint32_t)bw, 128u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool shape_ok(int H, int S, int D) {
  if (H < 0 || S < 0) return false;
  // int32 row indexing inside the kernels: H*S*D and rows of the cache fit
  if ((int64_t)H * S * (int64_t)D >= (int64_t)1 << 31) return false;
  return true;
}

}  // namespace

extern "C" int dt_set_wait_limit_ns(int64_t ns) {
  g_wait_limit_ns.store(ns < 0 ? 0 : ns);
  return DT_OK;
}

namespace {
int fused_step(const dt_plan_params* p, int32_t head_begin, int32_t head_count, const uint8_t* d_plan, const void* Q,
               const void* K, const void* V, float* cache_O, float* cache_L, float* R, void* O, float* L,
               int64_t* d_counters, int32_t* d_status, float* d_err, int err_all, void* stream);
}  // namespace

extern "C" int dt_attn_partial_fused_heads(const dt_plan_params* p, int32_t head_begin, int32_t head_count,
                                           const uint8_t* d_plan, const void* Q, const void* K, const void* V,
                                           float* cache_O, float* cache_L, float* R, void* O, float* L,
                                           int64_t* d_counters, int32_t* d_status, void* stream) {
  return fused_step(p, head_begin, head_count, d_plan, Q, K, V, cache_O, cache_L, R, O, L, d_counters, d_status,
                    nullptr, 0, stream);
}

extern "C" int dt_attn_partial_fused_tracked(const dt_plan_params* p, const uint8_t* d_plan, const void* Q,
                                             const void* K, const void* V, float* cache_O, float* cache_L, void* O,
                                             float* L, int64_t* d_counters, int32_t* d_status, float* d_err,
                                             int32_t err_all, void* stream) {
  if (!p || p->mode == DT_MODE_WINDOW || !d_err) return DT_ERR_INVALID;
  return fused_step(p, 0, p->H, d_plan, Q, K, V, cache_O, cache_L, nullptr, O, L, d_counters, d_status, d_err,
                    err_all, stream);
}

namespace {
int fused_step(const dt_plan_params* p, int32_t head_begin, int32_t head_count, const uint8_t* d_plan, const void* Q,
               const void* K, const void* V, float* cache_O, float* cache_L, float* R, void* O, float* L,
               int64_t* d_counters, int32_t* d_status, float* d_err, int err_all, void* stream) {
  if (!p || p->mode < DT_MODE_ALL_COMPUTE || p->mode > DT_MODE_ANCHOR) return DT_ERR_INVALID;
  const bool win = p->mode == DT_MODE_WINDOW;
  if (!shape_ok(p->H, p->S, p->D)) return DT_ERR_INVALID;
  if (win ? p->window < 1 : p->P < 1) return DT_ERR_INVALID;
  if (p->group < 0 || (win && p->group != 0)) return DT_ERR_INVALID;
  if (p->state_dtype != DT_STATE_F32 && p->state_dtype != DT_STATE_BF16) return DT_ERR_INVALID;
  if (win && p->state_dtype != DT_STATE_F32) return DT_ERR_INVALID;
  if (head_begin < 0 || head_count < 0 || head_begin > p->H - head_count) return DT_ERR_INVALID;
  if (p->D != 64 && p->D != 72 && p->D != 128) return DT_ERR_UNSUPPORTED;
  const int nseg = win ? 2 : (p->group > 0 ? 1 + dt::ceil_div(p->P, p->group) : p->P);
  if (nseg > 64) return DT_ERR_UNSUPPORTED;              // the kernel keeps a plan row as a 64-bit mask
  if (head_count == 0 || p->S == 0) return DT_OK;
  if (!d_plan || !Q || !K || !V || !O || !L || !d_status) return DT_ERR_INVALID;
  if (win ? !R : (!cache_O || !cache_L)) return DT_ERR_INVALID;
  const void* ptrs[] = {d_plan, Q, K, V, O, L, d_status};
  for (const void* q : ptrs)
    if (!aligned16(q)) return DT_ERR_UNSUPPORTED;
  if ((cache_O && !aligned16(cache_O)) || (cache_L && !aligned16(cache_L)) || (R && !aligned16(R)) ||
      (d_counters && !aligned16(d_counters)) || (d_err && !aligned16(d_err)))
    return DT_ERR_UNSUPPORTED;

  dt::Geom G = dt::make_geom(p->H, p->S, p->D, win ? 1 : p->P, win ? p->window : 0, win ? 0 : p->group);
  const int dp = p->D == 72 ? 80 : p->D;
  dt::AttnParams kp;
  memset(&kp, 0, sizeof(kp));
  const CUtensorMapSwizzle sw128 = CU_TENSOR_MAP_SWIZZLE_128B, sw32 = CU_TENSOR_MAP_SWIZZLE_32B;
  if (!encode_qkv(&kp.tmQ, Q, p->H, p->S, p->D, 64, sw128) || !encode_qkv(&kp.tmK, K, p->H, p->S, p->D, 64, sw128) ||
      !encode_qkv(&kp.tmV, V, p->H, p->S, p->D, 64, sw128))
    return DT_ERR_CUDA;
  if (p->D == 72) {
    if (!encode_qkv(&kp.tmQt, Q, p->H, p->S, p->D, 16, sw32) || !encode_qkv(&kp.tmKt, K, p->H, p->S, p->D, 16, sw32) ||
        !encode_qkv(&kp.tmVt, V, p->H, p->S, p->D, 16, sw32))
      return DT_ERR_CUDA;
  }
  kp.plan = d_plan;
  kp.cache_O = cache_O;
  kp.cache_L = cache_L;
  kp.R = R;
  kp.O = O;
  kp.L = L;
  kp.counters = d_counters;
  kp.status = d_status;
  kp.H = p->H; kp.S = p->S; kp.D = p->D; kp.P = win ? 1 : p->P; kp.window = win ? p->window : 0;
  kp.geom = G;
  kp.state_bf16 = p->state_dtype == DT_STATE_BF16;
  kp.cache_v8 = (reinterpret_cast<uintptr_t>(cache_O) & 31u) == 0;
  // items are numbered over all heads, so a head range computes exactly what
  // the whole launch computes for those heads
  kp.item0 = head_begin * G.nqt;
  kp.item_end = (head_begin + head_count) * G.nqt;
  kp.scale_log2 = (float)(1.4426950408889634 / sqrt((double)p->D));
  kp.wait_limit_ns = (uint64_t)g_wait_limit_ns.load();
  kp.err = d_err;
  kp.err_all = err_all ? 1 : 0;
  int sms = 0;
  if (int e = sm_count(&sms)) return e;
  const int n_items = kp.item_end - kp.item0;
  if (n_items == 0) return DT_OK;
  int grid = n_items < sms ? n_items : sms;
  return dt::launch_attn_fused(kp, dp, grid, reinterpret_cast<cudaStream_t>(stream));
}
}  // namespace

extern "C" int dt_attn_partial_fused(const dt_plan_params* p, const uint8_t* d_plan, const void* Q, const void* K,
                                     const void* V, float* cache_O, float* cache_L, float* R, void* O, float* L,
                                     int64_t* d_counters, int32_t* d_status, void* stream) {
  if (!p) return DT_ERR_INVALID;
  return dt_attn_partial_fused_heads(p, 0, p->H, d_plan, Q, K, V, cache_O, cache_L, R, O, L, d_counters, d_status,
                                     stream);
}

extern "C" int dt_state_merge(int32_t N, int32_t H, int32_t S, int32_t D, const float* O_in, const float* L_in,
                              float* O_out, float* L_out, int32_t* d_status, void* stream) {
  if (N < 1 || D < 4 || D % 4 != 0 || !shape_ok(H, S, D)) return DT_ERR_INVALID;
  if ((int64_t)N * H * S * (int64_t)D >= ((int64_t)1 << 40)) return DT_ERR_INVALID;
  if ((int64_t)H * S == 0) return DT_OK;
  if (!O_in || !L_in || !O_out || !L_out) return DT_ERR_INVALID;
  if (!aligned16(O_in) || !aligned16(O_out) || !aligned16(L_in) || !aligned16(L_out)) return DT_ERR_UNSUPPORTED;
  (void)d_status;
  int sms = 0;
  if (int e = sm_count(&sms)) return e;
  return dt::launch_state_merge(N, H, S, D, O_in, L_in, O_out, L_out, sms, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int dt_state_cache_update(const dt_plan_params* p, const uint8_t* d_plan, const float* fresh_O,
                                     const float* fresh_L, float* cache_O, float* cache_L, int32_t* d_status,
                                     void* stream) {
  if (!p || p->mode == DT_MODE_WINDOW || p->mode < DT_MODE_ALL_COMPUTE || p->mode > DT_MODE_ANCHOR)
    return DT_ERR_INVALID;
  if (p->P < 1 || p->group < 0 || p->D < 4 || p->D % 4 != 0 || !shape_ok(p->H, p->S, p->D)) return DT_ERR_INVALID;
  if (p->state_dtype != DT_STATE_F32) return DT_ERR_UNSUPPORTED;
  if (p->H == 0 || p->S == 0) return DT_OK;
  if (!d_plan || !fresh_O || !fresh_L || !cache_O || !cache_L) return DT_ERR_INVALID;
  if (!aligned16(fresh_O) || !aligned16(cache_O) || !aligned16(fresh_L) || !aligned16(cache_L))
    return DT_ERR_UNSUPPORTED;
  (void)d_status;
  dt::Geom G = dt::make_geom(p->H, p->S, p->D, p->P, 0, p->group);
  int sms = 0;
  if (int e = sm_count(&sms)) return e;
  return dt::launch_cache_update(G, d_plan, fresh_O, fresh_L, cache_O, cache_L, sms,
                                 reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int dt_group_compose(const dt_plan_params* p, int32_t factor, int32_t* stamps, float* cache_O,
                                float* cache_L, int32_t* d_status, void* stream) {
  if (!p || p->mode == DT_MODE_WINDOW || p->mode < DT_MODE_ALL_COMPUTE || p->mode > DT_MODE_ANCHOR)
    return DT_ERR_INVALID;
  if (p->P < 1 || p->group < 1 || factor < 2 || factor > 8) return DT_ERR_INVALID;
  if (p->state_dtype != DT_STATE_F32) return DT_ERR_UNSUPPORTED;
  if (p->D < 4 || p->D % 4 != 0 || !shape_ok(p->H, p->S, p->D)) return DT_ERR_INVALID;
  if ((int64_t)p->group * factor > (int64_t)1 << 30) return DT_ERR_INVALID;
  const dt::Geom G = dt::make_geom(p->H, p->S, p->D, p->P, 0, p->group);
  const int m = G.P - 1, m2 = dt::ceil_div(m, factor);
  if ((int64_t)p->H * p->S > 0) {
    if (!cache_O || !cache_L) return DT_ERR_INVALID;
    if (!aligned16(cache_O) || !aligned16(cache_L)) return DT_ERR_UNSUPPORTED;
  }
  (void)d_status;
  if (stamps) {
    // [nqt][1+m] -> [nqt][1+m2] in place, rows and entries in increasing
    // order with no buffer: new entry i of row qt lands at qt*(1+m2)+i, which
    // is never after old entry i of that row, and every old entry it could
    // cover (row < qt, or entry <= i of row qt) has already been consumed,
    // since new entry i reads old entries factor*i+1 .. > i.
    for (int qt = 0; qt < G.nqt; ++qt) {
      const int32_t* old_row = stamps + (size_t)qt * (1 + m);
      int32_t* new_row = stamps + (size_t)qt * (1 + m2);
      new_row[0] = old_row[0];
      for (int i = 0; i < m2; ++i) {
        int32_t s = old_row[1 + factor * i];
        for (int j = factor * i + 1; j < factor * i + factor && j < m; ++j) s = old_row[1 + j] < s ? old_row[1 + j] : s;
        new_row[1 + i] = s;
      }
    }
  }
  if ((int64_t)p->H * p->S == 0) return DT_OK;
  int sms = 0;
  if (int e = sm_count(&sms)) return e;
  return dt::launch_group_compose(m, factor, p->H, p->S, p->D, cache_O, cache_L, sms,
                                  reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int dt_state_importance(const dt_plan_params* p, const float* cache_L, const float* L, float* d_weights,
                                   int32_t* d_status, void* stream) {
  if (!p || p->mode == DT_MODE_WINDOW || p->mode < DT_MODE_ALL_COMPUTE || p->mode > DT_MODE_ANCHOR)
    return DT_ERR_INVALID;
  if (p->P < 1 || p->group < 0 || p->D < 1 || !shape_ok(p->H, p->S, p->D)) return DT_ERR_INVALID;
  const dt::Geom G = dt::make_geom(p->H, p->S, p->D, p->P, 0, p->group);
  if ((int64_t)G.nqt * G.P == 0) return DT_OK;
  if (!d_weights) return DT_ERR_INVALID;
  if (p->H == 0) return dt::launch_fill_zero(d_weights, (int64_t)G.nqt * G.P, reinterpret_cast<cudaStream_t>(stream));
  if (!cache_L || !L) return DT_ERR_INVALID;
  if (!aligned16(cache_L) || !aligned16(L) || !aligned16(d_weights)) return DT_ERR_UNSUPPORTED;
  (void)d_status;
  return dt::launch_state_importance(G, cache_L, L, d_weights, reinterpret_cast<cudaStream_t>(stream));
}

namespace {
bool overlap(const void* a, const void* b, size_t n) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + n && y < x + n;
}
}  // namespace

extern "C" int dt_share_output(int32_t n_heads, int32_t S, int32_t D, const void* src_O, const float* src_L,
                               void* dst_O, float* dst_L, void* stream) {
  if (n_heads < 0 || S < 0 || D < 1 || !shape_ok(n_heads, S, D)) return DT_ERR_INVALID;
  const size_t nO = (size_t)n_heads * S * D * 2, nL = (size_t)n_heads * S * 4;
  if (nO == 0) return DT_OK;
  if (!src_O || !src_L || !dst_O || !dst_L) return DT_ERR_INVALID;
  const bool sameO = src_O == dst_O, sameL = src_L == dst_L;
  if ((!sameO && overlap(src_O, dst_O, nO)) || (!sameL && overlap(src_L, dst_L, nL))) return DT_ERR_INVALID;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (!sameO && cudaMemcpyAsync(dst_O, src_O, nO, cudaMemcpyDeviceToDevice, st) != cudaSuccess) return DT_ERR_CUDA;
  if (!sameL && cudaMemcpyAsync(dst_L, src_L, nL, cudaMemcpyDeviceToDevice, st) != cudaSuccess) return DT_ERR_CUDA;
  return DT_OK;
}

extern "C" int dt_attn_cfg_shared(const dt_plan_params* p, const uint8_t* d_plan, const void* Q, const void* K,
                                  const void* V, float* cache_O, float* cache_L, float* R, void* O, float* L,
                                  int64_t* d_counters, int32_t* d_status, void* stream) {
  if (!p || p->H % 2 != 0) return DT_ERR_INVALID;
  const int hb = p->H / 2;
  if (int e = dt_attn_partial_fused_heads(p, 0, hb, d_plan, Q, K, V, cache_O, cache_L, R, O, L, d_counters, d_status,
                                          stream))
    return e;
  if (hb == 0 || p->S == 0) return DT_OK;
  const size_t half = (size_t)hb * p->S;
  if (int e = dt_share_output(hb, p->S, p->D, O, L, static_cast<uint16_t*>(O) + half * p->D, L + half, stream))
    return e;
  const bool win = p->mode == DT_MODE_WINDOW;
  const dt::Geom G = dt::make_geom(p->H, p->S, p->D, win ? 1 : p->P, win ? p->window : 0, win ? 0 : p->group);
  int sms = 0;
  if (int e = sm_count(&sms)) return e;
  const int elem = win ? 4 : (p->state_dtype == DT_STATE_BF16 ? 2 : 4);
  return dt::launch_share_states(G, d_plan, hb, elem, cache_O, cache_L, R, sms,
                                 reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int dt_window_residual(int32_t op, int32_t H, int32_t S, int32_t D, const float* O_full,
                                  const float* O_win, float* R, void* O, int32_t* d_status, void* stream) {
  if (op != DT_WR_MAKE && op != DT_WR_APPLY) return DT_ERR_INVALID;
  if (D < 4 || D % 4 != 0 || !shape_ok(H, S, D)) return DT_ERR_INVALID;
  const int64_t n = (int64_t)H * S * D;
  if (n == 0) return DT_OK;
  if (!O_win || !R || (op == DT_WR_MAKE && !O_full) || (op == DT_WR_APPLY && !O)) return DT_ERR_INVALID;
  if (!aligned16(O_win) || !aligned16(R) || (O_full && !aligned16(O_full)) || (O && !aligned16(O)))
    return DT_ERR_UNSUPPORTED;
  (void)d_status;
  int sms = 0;
  if (int e = sm_count(&sms)) return e;
  return dt::launch_window_residual(op, n, O_full, O_win, R, O, sms, reinterpret_cast<cudaStream_t>(stream));
}
