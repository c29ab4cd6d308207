// pi_attn.cu -- head-sparse decode self-attention: the operator behind the
// second per-layer predictor of the PowerInfer pages (unite.ai, "Adaptif
// Sparsite Predictor’ları": besides the FFN predictor each layer has one for
// its self-attention block, which picks the heads to compute).
//
// The head list is [0, n_hot) ++ head_idx[0, *head_count) -- made by
// pi_predict with the heads as its "neurons" -- and only those heads are
// touched: their rows of Wq, Wk, Wv, their positions of the KV cache, their
// rows of W_o^T.  Per call (a token block of B independent sequences):
//   k_attn_proj     q, k, v of the listed heads (one warp per weight row,
//                   fp32 accumulation); k and v also land in the cache at
//                   position len, in the cache's type
//   k_attn_decode   split softmax attention: CTA = (token, listed head,
//                   chunk of positions 0..len); each warp keeps a running
//                   max, sum and weighted value over its positions; the
//                   CTA's warps are merged and written as one partial
//   k_attn_combine  the chunks of a head merged in order -> the head's output
//                   o (fp32), plus the list of W_o^T rows (h dh + i) it feeds
//   k_ffn_down +    the output projection as a gathered-row product over
//   k_ffn_reduce    those rows (the FFN's down-projection kernels), y fp32
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "pi_attn.cuh"
#include "pi_common.cuh"
#include "pi_kernels_v1.cuh"

namespace pi {

namespace {

constexpr int kAttnNB = 4;  // tokens per pass of the projection warps

__device__ __forceinline__ int attn_list(const int32_t* head_count, int n_heads, int n_hot) {
  int c = *head_count;
  const int C = n_heads - n_hot;
  c = c < 0 ? 0 : (c > C ? C : c);
  return n_hot + c;
}

// head of list position p, or -1 for an entry outside [n_hot, n_heads)
__device__ __forceinline__ int attn_head(int p, int n_hot, int n_heads, const int32_t* head_idx) {
  if (p < n_hot) return p;
  const int h = __ldg(head_idx + (p - n_hot));
  return (h < n_hot || h >= n_heads) ? -1 : h;
}

template <int T>
__device__ __forceinline__ float ld_elem(const void* base, int64_t i) {
  if constexpr (T == kF32) return __ldg(reinterpret_cast<const float*>(base) + i);
  else return __half2float(reinterpret_cast<const __half*>(base)[i]);
}

template <int T>
__device__ __forceinline__ void st_elem(void* base, int64_t i, float v) {
  if constexpr (T == kF32) reinterpret_cast<float*>(base)[i] = v;
  else reinterpret_cast<__half*>(base)[i] = __float2half_rn(v);
}

// q, k, v rows of the listed heads: qkv[b][p][m][i] (m = 0 q, 1 k, 2 v) fp32;
// k and v are also stored in the cache at position len.
template <int WT, int XT, int CT>
__global__ void __launch_bounds__(256) k_attn_proj(const AttnParams p) {
  constexpr int E = Unit<WT>::E;
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int dh = p.d / p.n_heads;
  const int n_list = attn_list(p.head_count, p.n_heads, p.n_hot);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    const int c = *p.head_count;
    if (c < 0 || c > p.n_heads - p.n_hot) set_status(&p.ctrl->status, kStCapacity);
  }
  const int rows = n_list * 3 * dh;
  const int units = p.d / E;
  for (int r = gw; r < rows; r += nw) {
    const int pos = r / (3 * dh), m = (r / dh) % 3, i = r % dh;
    const int h = attn_head(pos, p.n_hot, p.n_heads, p.head_idx);
    if (h < 0) {
      if (lane == 0 && m == 0 && i == 0) set_status(&p.ctrl->status, kStIndex);
      continue;
    }
    const void* W = m == 0 ? p.Wq : (m == 1 ? p.Wk : p.Wv);
    const int64_t wrow = (int64_t)h * dh + i;
    for (int b0 = 0; b0 < p.B; b0 += kAttnNB) {
      const int nb = min(kAttnNB, p.B - b0);
      float acc[kAttnNB];
#pragma unroll
      for (int t = 0; t < kAttnNB; ++t) acc[t] = 0.f;
      for (int un = lane; un < units; un += 32) {
        float w[E];
        load_w_unit<WT>(W, nullptr, wrow, p.d, un, w);
#pragma unroll
        for (int t = 0; t < kAttnNB; ++t) {
          if (t < nb) {
            float x[E];
            load_h_unit<WT, XT>(p.x, b0 + t, p.d, un, x);
#pragma unroll
            for (int e = 0; e < E; ++e) acc[t] = fmaf(w[e], x[e], acc[t]);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < kAttnNB; ++t) acc[t] = warp_sum(acc[t]);
      if (lane == 0) {
        for (int t = 0; t < nb; ++t) {
          const int b = b0 + t;
          p.qkv[(((int64_t)b * p.n_heads + pos) * 3 + m) * dh + i] = acc[t];
          if (m > 0) {
            void* cache = m == 1 ? p.K : p.V;
            st_elem<CT>(cache, (((int64_t)b * p.n_heads + h) * p.s_max + p.len) * dh + i, acc[t]);
          }
        }
      }
    }
  }
}

// One chunk of positions of one (token, listed head): partial max, sum and
// weighted value.  Lanes hold dh / 32 consecutive elements of q and of each
// position's key and value; warp w takes positions t0 + w, t0 + w + 4, ...
template <int CT, int EPL>
__global__ void __launch_bounds__(128) k_attn_decode(const AttnParams p) {
  __shared__ float sm_m[4], sm_l[4];
  __shared__ float sm_o[4][32 * EPL];
  const int split = blockIdx.x, pos = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int dh = 32 * EPL;
  const int n_list = attn_list(p.head_count, p.n_heads, p.n_hot);
  if (pos >= n_list) return;
  const int h = attn_head(pos, p.n_hot, p.n_heads, p.head_idx);
  float* out = p.part + (((int64_t)b * p.n_heads + pos) * p.nsplit + split) * (dh + 4);
  const int total = p.len + 1;
  const int chunk = (total + p.nsplit - 1) / p.nsplit;
  const int t0 = split * chunk, t1 = min(total, t0 + chunk);
  float m = -INFINITY, l = 0.f, o[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) o[e] = 0.f;
  if (h >= 0 && t0 < t1) {
    const float* qkv = p.qkv + (((int64_t)b * p.n_heads + pos) * 3) * dh;
    const float scale = rsqrtf((float)dh);
    float q[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) q[e] = qkv[lane * EPL + e] * scale;
    const int64_t crow = ((int64_t)b * p.n_heads + h) * p.s_max;
    for (int t = t0 + warp; t < t1; t += 4) {
      float kv[EPL], vv[EPL];
      if (t < p.len) {
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          kv[e] = ld_elem<CT>(p.K, (crow + t) * dh + lane * EPL + e);
          vv[e] = ld_elem<CT>(p.V, (crow + t) * dh + lane * EPL + e);
        }
      } else {  // the new token: this step's own k and v
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          kv[e] = qkv[dh + lane * EPL + e];
          vv[e] = qkv[2 * dh + lane * EPL + e];
        }
      }
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) s = fmaf(q[e], kv[e], s);
      s = warp_sum(s);
      const float mn = fmaxf(m, s);
      const float alpha = expf(m - mn), beta = expf(s - mn);
      l = l * alpha + beta;
#pragma unroll
      for (int e = 0; e < EPL; ++e) o[e] = fmaf(o[e], alpha, beta * vv[e]);
      m = mn;
    }
  }
  if (lane == 0) {
    sm_m[warp] = m;
    sm_l[warp] = l;
  }
#pragma unroll
  for (int e = 0; e < EPL; ++e) sm_o[warp][lane * EPL + e] = o[e];
  __syncthreads();
  if (warp == 0) {
    float M = sm_m[0];
    for (int w = 1; w < 4; ++w) M = fmaxf(M, sm_m[w]);
    float L = 0.f, O[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) O[e] = 0.f;
    for (int w = 0; w < 4; ++w) {
      const float f = sm_m[w] == -INFINITY ? 0.f : expf(sm_m[w] - M);
      L = fmaf(sm_l[w], f, L);
#pragma unroll
      for (int e = 0; e < EPL; ++e) O[e] = fmaf(sm_o[w][lane * EPL + e], f, O[e]);
    }
    if (lane == 0) {
      out[dh] = M;
      out[dh + 1] = L;
    }
#pragma unroll
    for (int e = 0; e < EPL; ++e) out[lane * EPL + e] = O[e];
  }
}

// Merge the chunks of each (token, listed head) in chunk order -> a[b][pos*dh + i]
// (the activations of the output projection), and the W_o^T row of each of
// them (-1 for an invalid head: the projection skips it).
__global__ void __launch_bounds__(256) k_attn_combine(const AttnParams p, float* a, int32_t* orow, int32_t* ocount) {
  const int pos = blockIdx.x, b = blockIdx.y, i = threadIdx.x;
  const int dh = p.d / p.n_heads;
  const int n_list = attn_list(p.head_count, p.n_heads, p.n_hot);
  if (pos == 0 && b == 0 && i == 0) *ocount = n_list * dh;
  if (pos >= n_list || i >= dh) return;
  const int h = attn_head(pos, p.n_hot, p.n_heads, p.head_idx);
  const float* part = p.part + (((int64_t)b * p.n_heads + pos) * p.nsplit) * (dh + 4);
  float M = -INFINITY;
  for (int s = 0; s < p.nsplit; ++s) M = fmaxf(M, __ldcg(part + s * (dh + 4) + dh));
  float L = 0.f, O = 0.f;
  for (int s = 0; s < p.nsplit; ++s) {
    const float ms = __ldcg(part + s * (dh + 4) + dh);
    const float f = ms == -INFINITY ? 0.f : expf(ms - M);
    L = fmaf(__ldcg(part + s * (dh + 4) + dh + 1), f, L);
    O = fmaf(__ldcg(part + s * (dh + 4) + i), f, O);
  }
  a[(int64_t)b * p.d + pos * dh + i] = (h >= 0 && L > 0.f) ? O / L : 0.f;
  if (b == 0) orow[pos * dh + i] = h >= 0 ? h * dh + i : -1;
}

template <int WT, int XT, int CT>
cudaError_t launch_proj_t(const AttnParams& p, int sms, cudaStream_t st) {
  const int dh = p.d / p.n_heads;
  const int rows = p.n_heads * 3 * dh;  // upper bound: every head listed
  const int grid = min((rows + 7) / 8, sms * 8);
  k_attn_proj<WT, XT, CT><<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

template <int CT>
cudaError_t launch_decode_t(const AttnParams& p, cudaStream_t st) {
  const int dh = p.d / p.n_heads;
  const dim3 grid(p.nsplit, p.n_heads, p.B);
  switch (dh / 32) {
    case 1: k_attn_decode<CT, 1><<<grid, 128, 0, st>>>(p); break;
    case 2: k_attn_decode<CT, 2><<<grid, 128, 0, st>>>(p); break;
    case 4: k_attn_decode<CT, 4><<<grid, 128, 0, st>>>(p); break;
    case 8: k_attn_decode<CT, 8><<<grid, 128, 0, st>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

bool attn_head_dim_ok(int dh) { return dh == 32 || dh == 64 || dh == 128 || dh == 256; }

int attn_splits(int len, int B, int n_heads, int sms) {
  // about 128 positions per chunk, and enough CTAs to cover the SMs twice
  int s = (len + 1 + 127) / 128;
  const int fill = (2 * sms + B * n_heads - 1) / (B * n_heads);
  if (s < fill) s = fill;
  if (s > len + 1) s = len + 1;
  if (s > kAttnMaxSplit) s = kAttnMaxSplit;
  return s < 1 ? 1 : s;
}

cudaError_t launch_attention(const AttnParams& p, int wtype, int xtype, int ctype, float* a, int32_t* orow,
                             int32_t* ocount, float* partial, int G, float* y, int sms, cudaStream_t st) {
  cudaError_t e;
#define PI_PROJ(W_, X_, C_) \
  if (wtype == W_ && xtype == X_ && ctype == C_) e = launch_proj_t<W_, X_, C_>(p, sms, st); else
  PI_PROJ(kF16, kF16, kF16) PI_PROJ(kF16, kF16, kF32) PI_PROJ(kF32, kF32, kF32) PI_PROJ(kF32, kF32, kF16)
  PI_PROJ(kF32, kF16, kF16) PI_PROJ(kF32, kF16, kF32)
  return cudaErrorInvalidValue;
#undef PI_PROJ
  if (e != cudaSuccess) return e;
  e = ctype == kF16 ? launch_decode_t<kF16>(p, st) : launch_decode_t<kF32>(p, st);
  if (e != cudaSuccess) return e;
  const int dh = p.d / p.n_heads;
  k_attn_combine<<<dim3(p.n_heads, p.B), dh, 0, st>>>(p, a, orow, ocount);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // output projection: the listed heads' rows of W_o^T, weighted by o
  if ((e = launch_ffn_down(wtype, p.B, p.d, p.d, 0, orow, ocount, p.WoT, nullptr, a, p.d, partial, G, st)) !=
      cudaSuccess)
    return e;
  return launch_ffn_reduce(partial, G, p.B, p.d, nullptr, y, st);
}

}  // namespace pi
