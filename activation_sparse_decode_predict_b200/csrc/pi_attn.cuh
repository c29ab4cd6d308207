// pi_attn.cuh -- launcher of the head-sparse decode self-attention (pi_attn.cu).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "pi_common.cuh"

namespace pi {

constexpr int kAttnMaxSplit = 64;  // chunks of cache positions per (token, head) at most

struct AttnParams {
  int d, n_heads, n_hot, B, s_max, len, nsplit;
  const void* x;            // [B, d] token block
  const int32_t* head_idx;  // predicted heads (list positions n_hot ..)
  const int32_t* head_count;
  const void *Wq, *Wk, *Wv, *WoT;  // [d, d] each, head h = rows h*dh .. h*dh+dh-1
  void *K, *V;              // caches [B, n_heads, s_max, dh]
  float* qkv;               // [B, n_heads, 3, dh] q, k, v of the listed heads (by list position)
  float* part;              // [B, n_heads, nsplit, dh + 4] chunk partials: o, max, sum
  Ctrl* ctrl;
};

// head dimensions the kernels take (one to eight values per lane)
bool attn_head_dim_ok(int dh);
// chunks of the len + 1 positions of each (token, head)
int attn_splits(int len, int B, int n_heads, int sms);
// q/k/v (+ cache append), split attention, merge, output projection -> y [B, d] fp32;
// a [B, d], orow [d], ocount, partial [G, B, d]: scratch
cudaError_t launch_attention(const AttnParams& p, int wtype, int xtype, int ctype, float* a, int32_t* orow,
                             int32_t* ocount, float* partial, int G, float* y, int sms, cudaStream_t st);

}  // namespace pi
