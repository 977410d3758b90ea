// state_ops.h -- launchers of the HBM-bound state kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "geometry.h"

namespace dt {

int launch_state_merge(int N, int H, int S, int D, const float* O_in, const float* L_in, float* O_out,
                       float* L_out, int sms, cudaStream_t st);
int launch_cache_update(const Geom& G, const uint8_t* plan, const float* fO, const float* fL, float* cO, float* cL,
                        int sms, cudaStream_t st);
int launch_group_compose(int m, int factor, int H, int S, int D, float* cO, float* cL, int sms, cudaStream_t st);
int launch_state_importance(const Geom& G, const float* cL, const float* L, float* w, cudaStream_t st);
int launch_fill_zero(float* x, int64_t n, cudaStream_t st);
int launch_share_states(const Geom& G, const uint8_t* plan, int hb, int elem_bytes, void* cO, float* cL, float* R,
                        int sms, cudaStream_t st);
int launch_window_residual(int op, int64_t n, const float* Of, const float* Ow, float* R, void* O, int sms,
                           cudaStream_t st);

}  // namespace dt
