// attn_fused.h -- kernel parameter block and launcher of the fused kernel.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "geometry.h"

namespace dt {

struct AttnParams {
  CUtensorMap tmQ, tmK, tmV;        // 64-column blocks, 128-byte swizzle
  CUtensorMap tmQt, tmKt, tmVt;     // 16-column tail block (D = 72), 32-byte swizzle
  const uint8_t* plan;              // [nqt][nseg]
  float* cache_O;
  float* cache_L;
  float* R;
  void* O;
  float* L;
  int64_t* counters;
  int32_t* status;
  int H, S, D, P, window;           // P: partitions (ignored in window mode)
  Geom geom;                        // make_geom(H, S, D, P, window), read from the parameter bank
  int item0, item_end;              // items [item0, item_end) of the H * nqt (head-major) items
  int state_bf16;                   // cached OUT is bf16 (cache_O then points to bf16 data)
  int cache_v8;                     // cache_O is 32-byte aligned (fp32 states stored 32 bytes at a time)
  float scale_log2;                 // log2(e) / sqrt(D)
  float* err;                       // state errors [nqt][nseg][H][4][2] (tracked step) or null
  int err_all;                      // measure every computed key set (else only the local one)
  uint64_t wait_limit_ns;
};

// Dynamic shared memory of the kernel instance for padded head dim dp.
int attn_fused_smem_bytes(int dp);
// Launch the instance for padded head dim dp (64, 80, 128) on `grid` CTAs.
int launch_attn_fused(const AttnParams& kp, int dp, int grid, cudaStream_t stream);

}  // namespace dt
