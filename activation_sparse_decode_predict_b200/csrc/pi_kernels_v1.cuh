// pi_kernels_v1.cuh -- launchers of the stand-alone libpi kernels.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace pi {

// ptype: fp32, fp16 or Q4_0 predictor matrices (Q4_0: scales in P1_sc / P2_sc, else unused)
cudaError_t launch_pred_u(int ptype, const void* P1, const void* P1_sc, const void* h, int B, int d, int r, float* u,
                          int sms, cudaStream_t st);
cudaError_t launch_pred_score(int ptype, const void* P2, const void* P2_sc, const float* bp, const float* u, int B,
                              int r, int C, float thr, uint32_t* tile_mask, int* tile_count, cudaStream_t st);
cudaError_t launch_compact(const uint32_t* tile_mask, const int* tile_count, int C, int n_hot, int32_t* idx,
                           int32_t* count, cudaStream_t st);
cudaError_t launch_ffn_act(int wtype, int htype, int act, const void* h, int B, int d, int ffn, int n_hot,
                           const int32_t* idx, const int32_t* count, const void* wg, const void* wg_sc,
                           const void* wu, const void* wu_sc, const float* b1, float* a, int n_max, int* status,
                           int sms, cudaStream_t st);
// position ranges (split-K partials, at most kGMax) of the down projection
int down_ranges(int d, int sms);
// down projection of the listed rows into G split-K partials; the activations
// come from a [B][n_max], or with `pre` from the token-block gate/up dots
// (pre [pre_S][pre_R][2][B]) and b1 with activation kind `act`
cudaError_t launch_ffn_down(int wtype, int B, int d, int ffn, int n_hot, const int32_t* idx, const int32_t* count,
                            const void* wd, const void* wd_sc, const float* a, int n_max, float* partial, int G,
                            cudaStream_t st, const float* pre = nullptr, int pre_S = 0, int pre_R = 0,
                            const float* b1 = nullptr, int act = 0);
cudaError_t launch_ffn_reduce(const float* partial, int G, int B, int d, const float* b2, float* y,
                              cudaStream_t st);
cudaError_t launch_rmsnorm(int htype, const void* h, const float* y, int B, int d, float eps, void* h_out,
                           cudaStream_t st);

}  // namespace pi
