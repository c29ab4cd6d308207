// pi_batch.cuh -- launchers of the tensor-core sparse FFN for token blocks of
// kBatchMin..16 tokens (fp16 tokens; fp16 weights, or Q4_0 gate/up rows on
// the tensor cores with the down projection on the CUDA cores).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "pi_common.cuh"

namespace pi {

constexpr int kBatchMin = 3;  // smaller blocks: the CUDA-core kernels

// true if the shape takes the tensor-core path (htype: the token type)
bool batch_supported(int wtype, int htype, int d, int B);
// true if the predictor of the block takes the tensor-core path
bool batch_pred_supported(int ptype, int d, int r, int B);
// bytes of the pre-activation buffer ([parts <= 4][ffn][2][B] fp32)
size_t batch_pre_bytes(int ffn, int B);
// neuron ranges of the down kernel (= split-K partial slots it writes)
int batch_ranges(int d, int sms);
// u = ReLU(P1 h) (dots -> upre [parts][r][B]), scores of P2 against u split
// into fp16 hi + lo rows -> sc [parts][C][2B], threshold -> the compaction's tile masks
cudaError_t launch_batch_predict(const void* h, int B, int d, int r, int C, int n_hot, const void* P1,
                                 const void* P2, const float* bp, float thr, float* upre, float* sc,
                                 uint32_t* tile_mask, int* tile_count, Ctrl* ctrl, int sms, cudaStream_t st);
// gate/up dots -> pre, then activations + down -> partial[ranges][B][d]
// (NR ranges: batch_ranges for fp16 weights, down_ranges for Q4_0; *_sc:
// the Q4_0 scales, else unused)
cudaError_t launch_batch_ffn(int act, int wtype, const void* h, int B, int d, int ffn, int n_hot, const int32_t* idx,
                             const int32_t* count, const void* wg, const void* wg_sc, const void* wu,
                             const void* wu_sc, const void* wd, const void* wd_sc, const float* b1, float* pre,
                             float* partial, int NR, Ctrl* ctrl, int sms, cudaStream_t st);

}  // namespace pi
