// pi_batch.cuh -- launchers of the tensor-core sparse FFN for token blocks of
// kBatchMin..16 tokens (fp16 weights and tokens).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "pi_common.cuh"

namespace pi {

constexpr int kBatchMin = 3;  // smaller blocks: the CUDA-core kernels

// true if the shape takes the tensor-core path
bool batch_supported(int wtype, int ptype, int d, int B);
// bytes of the pre-activation buffer ([parts <= 4][ffn][2][B] fp32)
size_t batch_pre_bytes(int ffn, int B);
// neuron ranges of the down kernel (= split-K partial slots it writes)
int batch_ranges(int d, int sms);
// gate/up dots -> pre, then activations + down -> partial[ranges][B][d]
cudaError_t launch_batch_ffn(int act, const void* h, int B, int d, int ffn, int n_hot, const int32_t* idx,
                             const int32_t* count, const void* wg, const void* wu, const void* wd, const float* b1,
                             float* pre, float* partial, int NR, Ctrl* ctrl, int sms, cudaStream_t st);

}  // namespace pi
