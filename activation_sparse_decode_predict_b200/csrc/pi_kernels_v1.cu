// pi_kernels_v1.cu -- the stand-alone kernels behind pi_predict, pi_sparse_ffn
// and pi_residual_rmsnorm (sm_100a).  Each step is its own launch; the fused
// multi-layer path lives in pi_stack.cu.
//
// Pages: unite.ai "PowerInfer: Tüketici Düzeyinde bir GPU ile Hızlı Büyük Dil
// Modeli Sunucusu" -- "Adaptif Sparsite Predictor’ları" (predictor),
// "Nöron Bilinçli Operatör" (row/column operators); GeekNews "Serving model
// bahasa besar ...", "Keterbatasan dan FAQ" (ReLU, ReGLU, squared ReLU).
#include "pi_common.cuh"
#include "pi_kernels_v1.cuh"
#include "pi_launch.h"
#include "pi_layout.h"

namespace pi {

// ---------------------------------------------------------------------------
// Predictor step 1: u[b,k] = max(0, P1[k,:] . h[b,:]), fp32.  One warp per row.
// PT: predictor matrix type (fp32, fp16 or Q4_0 with its scales in P1_sc); the
// token block is fp32 with fp32 predictors and fp16 otherwise.
template <int PT, int NB>
__global__ void __launch_bounds__(256) k_pred_u(const void* __restrict__ P1, const void* __restrict__ P1_sc,
                                                const void* __restrict__ h, int B, int d, int r,
                                                float* __restrict__ u) {
  constexpr int E = Unit<PT>::E;
  constexpr int HT = PT == kF32 ? kF32 : kF16;
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int units = d / E;
  for (int k = gw; k < r; k += nw) {
    for (int b0 = 0; b0 < B; b0 += NB) {
      const int nb = min(NB, B - b0);
      float acc[NB];
#pragma unroll
      for (int i = 0; i < NB; ++i) acc[i] = 0.f;
      for (int un = lane; un < units; un += 32) {
        float w[E];
        load_w_unit<PT>(P1, P1_sc, k, d, un, w);
#pragma unroll
        for (int i = 0; i < NB; ++i) {
          if (i < nb) {
            float x[E];
            load_h_unit<PT, HT>(h, b0 + i, d, un, x);
#pragma unroll
            for (int e = 0; e < E; ++e) acc[i] = fmaf(w[e], x[e], acc[i]);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < NB; ++i) acc[i] = warp_sum(acc[i]);
      if (lane == 0) {
        for (int i = 0; i < nb; ++i) u[(int64_t)(b0 + i) * r + k] = fmaxf(acc[i], 0.f);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Predictor step 2: scores of one tile of 256 cold neurons (8 warps x 32 rows),
// s = P2[c,:] . u[b,:] + bp[c]; active = OR_b (s > thr).  Writes the tile's
// 8 ballot words and its popcount.
template <int PT, int NB>
__global__ void __launch_bounds__(256) k_pred_score(const void* __restrict__ P2, const void* __restrict__ P2_sc,
                                                    const float* __restrict__ bp,
                                                    const float* __restrict__ u, int B, int r, int C, float thr,
                                                    uint32_t* __restrict__ tile_mask, int* __restrict__ tile_count) {
  constexpr int E = Unit<PT>::E;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int units = r / E;
  bool mine = false;
  const int c_base = blockIdx.x * 256 + warp * 32;
  for (int t = 0; t < 32; ++t) {
    const int c = c_base + t;
    if (c >= C) break;
    const float bias = bp ? __ldg(bp + c) : 0.f;
    bool on = false;
    for (int b0 = 0; b0 < B; b0 += NB) {
      const int nb = min(NB, B - b0);
      float acc[NB];
#pragma unroll
      for (int i = 0; i < NB; ++i) acc[i] = 0.f;
      for (int un = lane; un < units; un += 32) {
        float w[E];
        load_w_unit<PT>(P2, P2_sc, c, r, un, w);
#pragma unroll
        for (int i = 0; i < NB; ++i) {
          if (i < nb) {
            float x[E];
            load_h_unit<PT, kF32>(u, b0 + i, r, un, x);
#pragma unroll
            for (int e = 0; e < E; ++e) acc[i] = fmaf(w[e], x[e], acc[i]);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < NB; ++i) {
        const float s = warp_sum(acc[i]) + bias;
        on |= (i < nb) && (s > thr);
      }
    }
    if (lane == t) mine = on;
  }
  const unsigned m = __ballot_sync(0xffffffffu, mine);
  __shared__ int cnt[8];
  if (lane == 0) {
    tile_mask[blockIdx.x * 8 + warp] = m;
    cnt[warp] = __popc(m);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int s = 0;
    for (int w = 0; w < 8; ++w) s += cnt[w];
    tile_count[blockIdx.x] = s;
  }
}

// ---------------------------------------------------------------------------
// Order-preserving compaction: one CTA per tile.  Each CTA sums the counts of
// the tiles before it (no inter-CTA waiting), then writes its tile's active
// rows in ascending order.  CTA 0 also writes the total count.
__global__ void __launch_bounds__(256) k_compact(const uint32_t* tile_mask,
                                                 const int* tile_count, int n_tiles, int n_hot,
                                                 int32_t* __restrict__ idx, int32_t* __restrict__ count) {
  __shared__ int red[8];
  __shared__ int wpre[9];
  pdl_trigger();
  pdl_wait();
  const int tile = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int before = 0, total = 0;
  for (int t = threadIdx.x; t < n_tiles; t += blockDim.x) {
    const int c = __ldcg(tile_count + t);
    total += c;
    if (t < tile) before += c;
  }
  // block reduce of `before` (and of `total` for CTA 0)
  for (int o = 16; o > 0; o >>= 1) {
    before += __shfl_xor_sync(0xffffffffu, before, o);
    total += __shfl_xor_sync(0xffffffffu, total, o);
  }
  __shared__ int redt[8];
  if (lane == 0) { red[warp] = before; redt[warp] = total; }
  const uint32_t m = __ldcg(tile_mask + tile * 8 + warp);
  if (threadIdx.x == 0) {
    wpre[0] = 0;
    for (int w = 0; w < 8; ++w) wpre[w + 1] = wpre[w] + __popc(__ldcg(tile_mask + tile * 8 + w));
  }
  __syncthreads();
  int base = 0, tot = 0;
  for (int w = 0; w < 8; ++w) { base += red[w]; tot += redt[w]; }
  if ((m >> lane) & 1u) {
    const int pos = base + wpre[warp] + __popc(m & ((1u << lane) - 1u));
    idx[pos] = n_hot + tile * 256 + warp * 32 + lane;
  }
  if (tile == 0 && threadIdx.x == 0) *count = tot;
}

// ---------------------------------------------------------------------------
// Sparse FFN step 1: activation of every listed neuron, one warp per neuron.
// list = [0, n_hot) ++ idx[0, count); a[b, p] for list position p.  A lane
// loads kActU units of the up (and gate) row before it decodes any of them.
constexpr int kActU = 4;

template <int WT, int HT, int ACT, int NB>
__global__ void __launch_bounds__(256) k_ffn_act(const void* __restrict__ h, int B, int d, int ffn, int n_hot,
                                                 const int32_t* __restrict__ idx, const int32_t* __restrict__ count,
                                                 const void* __restrict__ wg, const void* __restrict__ wg_sc,
                                                 const void* __restrict__ wu, const void* __restrict__ wu_sc,
                                                 const float* __restrict__ b1, float* __restrict__ a, int n_max,
                                                 int* __restrict__ status) {
  constexpr int E = Unit<WT>::E;
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int n_cold = ffn - n_hot;
  int cnt = *count;
  if (cnt < 0 || cnt > n_cold) {
    if (gw == 0 && lane == 0) set_status(status, kStCapacity);
    cnt = cnt < 0 ? 0 : n_cold;
  }
  const int n = n_hot + cnt;
  const int units = d / E;
  for (int p = gw; p < n; p += nw) {
    const int j = p < n_hot ? p : idx[p - n_hot];
    if (p >= n_hot && (j < n_hot || j >= ffn)) {
      if (lane == 0) set_status(status, kStIndex);
      if (lane < B) a[(int64_t)lane * n_max + p] = 0.f;
      continue;
    }
    const float bias = b1 ? __ldg(b1 + j) : 0.f;
    for (int b0 = 0; b0 < B; b0 += NB) {
      const int nb = min(NB, B - b0);
      float g[NB], v[NB];
#pragma unroll
      for (int i = 0; i < NB; ++i) { g[i] = 0.f; v[i] = 0.f; }
      for (int u0 = lane; u0 < units; u0 += 32 * kActU) {
        WRaw<WT> ru[kActU], rg[kActU];
#pragma unroll
        for (int k = 0; k < kActU; ++k) {
          const int un = u0 + 32 * k;
          if (un < units) {
            ru[k] = load_w_raw<WT>(wu, wu_sc, j, d, un);
            if constexpr (ACT == kReglu) rg[k] = load_w_raw<WT>(wg, wg_sc, j, d, un);
          }
        }
#pragma unroll
        for (int k = 0; k < kActU; ++k) {
          const int un = u0 + 32 * k;
          if (un < units) {
            float wu_[E], wg_[E];
            decode_w<WT>(ru[k], wu_);
            if constexpr (ACT == kReglu) decode_w<WT>(rg[k], wg_);
#pragma unroll
            for (int i = 0; i < NB; ++i) {
              if (i < nb) {
                float x[E];
                load_h_unit<WT, HT>(h, b0 + i, d, un, x);
#pragma unroll
                for (int e = 0; e < E; ++e) {
                  v[i] = fmaf(wu_[e], x[e], v[i]);
                  if constexpr (ACT == kReglu) g[i] = fmaf(wg_[e], x[e], g[i]);
                }
              }
            }
          }
        }
      }
#pragma unroll
      for (int i = 0; i < NB; ++i) {
        v[i] = warp_sum(v[i]);
        if constexpr (ACT == kReglu) g[i] = warp_sum(g[i]);
      }
      if (lane == 0) {
        for (int i = 0; i < nb; ++i) {
          float av;
          if constexpr (ACT == kReglu) av = activation<ACT>(g[i] + bias, v[i]);
          else av = activation<ACT>(v[i] + bias, 0.f);
          a[(int64_t)(b0 + i) * n_max + p] = av;
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Sparse FFN step 2: down projection.  CTA (c, r) covers chunk c of d -- 32
// lanes x 16 columns, a lane owning the same columns in every row -- for the
// list positions of range r (contiguous and balanced over the ranges).  The
// range's rows and activations are staged in shared memory; the 8 warps take
// its positions in turn with kDnU rows in flight per lane, and their sums are
// added in warp order through shared memory into the fp32 partial y[r]
// [B, d] (zeros for an empty range).  With `pre` the activations are made
// while staging, from the gate/up dots of the token-block row-dot kernel
// (pre [parts][pre_R][2][B], the parts added in order) and b1.
constexpr int kDnWarps = 8;
constexpr int kDnU = 4;
constexpr int kDnCap = 1024;  // positions staged at a time

template <int WT, int NB>
__global__ void __launch_bounds__(kDnWarps * 32) k_ffn_down(int B, int d, int ffn, int n_hot,
                                                            const int32_t* __restrict__ idx,
                                                            const int32_t* __restrict__ count,
                                                            const void* __restrict__ wd, const void* __restrict__ wd_sc,
                                                            const float* __restrict__ a, int n_max,
                                                            float* __restrict__ partial, const float* __restrict__ pre,
                                                            int pre_S, int pre_R, const float* __restrict__ b1,
                                                            int act) {
  constexpr int E = Unit<WT>::E;
  constexpr int UPT = 16 / E;      // units per lane
  constexpr int V = 16 * NB;       // sums per lane
  extern __shared__ float dsm[];
  int* srow = reinterpret_cast<int*>(dsm);  // [kDnCap] rows of the staged positions
  float* sact = dsm + kDnCap;               // [NB][kDnCap] their activations
  float* red = dsm;                         // [warps][V][32] after the stream (aliases the staging)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x, r = blockIdx.y, R = gridDim.y;
  const int n_cold = ffn - n_hot;
  int cnt = *count;
  cnt = cnt < 0 ? 0 : (cnt > n_cold ? n_cold : cnt);
  const int64_t n = n_hot + cnt;
  const int p0 = (int)(n * r / R), p1 = (int)(n * (r + 1) / R);
  const int units = d / E;
  const int ub = c * 32 * UPT + lane;  // this lane's first unit
  for (int b0 = 0; b0 < B; b0 += NB) {
    const int nb = min(NB, B - b0);
    float acc[UPT][E][NB];
    float corr[NB];  // Q4_0: the sum of 24 s a over the rows, taken off every column at the end
#pragma unroll
    for (int q = 0; q < UPT; ++q)
#pragma unroll
      for (int e = 0; e < E; ++e)
#pragma unroll
        for (int i = 0; i < NB; ++i) acc[q][e][i] = 0.f;
#pragma unroll
    for (int i = 0; i < NB; ++i) corr[i] = 0.f;
    for (int s0 = p0; s0 < p1; s0 += kDnCap) {
      const int len = min(kDnCap, p1 - s0);
      __syncthreads();  // the previous segment (or reduction) is done with the buffer
      for (int i = threadIdx.x; i < len; i += blockDim.x) {
        const int p = s0 + i;
        const int j = p < n_hot ? p : idx[p - n_hot];
        const bool ok = p < n_hot || (j >= n_hot && j < ffn);  // a bad entry is flagged by k_ffn_act
        srow[i] = ok ? j : 0;
        if (pre) {
          const float bias = (ok && b1) ? b1[j] : 0.f;
#pragma unroll
          for (int q = 0; q < NB; ++q) {
            float g = 0.f, v = 0.f;
            if (ok && q < nb) {
              for (int sp = 0; sp < pre_S; ++sp) {
                const float* pp = pre + ((int64_t)sp * pre_R + p) * 2 * B + b0 + q;
                g += pp[0];
                v += pp[B];
              }
            }
            sact[q * kDnCap + i] =
                !(ok && q < nb) ? 0.f : (act == kReglu ? act_eval(kReglu, g + bias, v) : act_eval(act, v + bias, 0.f));
          }
        } else {
#pragma unroll
          for (int q = 0; q < NB; ++q) sact[q * kDnCap + i] = (ok && q < nb) ? a[(int64_t)(b0 + q) * n_max + p] : 0.f;
        }
      }
      __syncthreads();
      for (int m0 = warp; m0 < len; m0 += kDnWarps * kDnU) {
        WRaw<WT> raw[kDnU][UPT] = {};
#pragma unroll
        for (int k = 0; k < kDnU; ++k) {
          const int m = m0 + kDnWarps * k;
          if (m < len) {
            const int j = srow[m];
#pragma unroll
            for (int q = 0; q < UPT; ++q)
              if (ub + 32 * q < units) raw[k][q] = load_w_raw<WT>(wd, wd_sc, j, d, ub + 32 * q);
          }
        }
#pragma unroll
        for (int k = 0; k < kDnU; ++k) {
          const int m = m0 + kDnWarps * k;
          if (m < len) {
            float av[NB];
#pragma unroll
            for (int i = 0; i < NB; ++i) av[i] = sact[i * kDnCap + m];
#pragma unroll
            for (int q = 0; q < UPT; ++q) {
              if (ub + 32 * q < units) {
                if constexpr (WT == kQ4_0) {
                  // s (q - 8) = 16 s f - 24 s with f = 1 + q / 16, made by setting
                  // the exponent bits of 1.0 around the nibble (exact)
                  const WRaw<WT>& r = raw[k][q];
                  const float sc = half_bits_to_float(r.s);
                  float as[NB];
#pragma unroll
                  for (int i = 0; i < NB; ++i) {
                    as[i] = 16.f * sc * av[i];
                    corr[i] = fmaf(24.f * sc, av[i], corr[i]);
                  }
                  float f[16];
#pragma unroll
                  for (int kk = 0; kk < 4; ++kk) {
                    f[kk] = __uint_as_float(0x3f800000u | (((r.q.x >> (8 * kk)) << 19) & 0x00780000u));
                    f[4 + kk] = __uint_as_float(0x3f800000u | (((r.q.y >> (8 * kk)) << 19) & 0x00780000u));
                    f[8 + kk] = __uint_as_float(0x3f800000u | (((r.q.x >> (8 * kk)) << 15) & 0x00780000u));
                    f[12 + kk] = __uint_as_float(0x3f800000u | (((r.q.y >> (8 * kk)) << 15) & 0x00780000u));
                  }
#pragma unroll
                  for (int e = 0; e < E; ++e)
#pragma unroll
                    for (int i = 0; i < NB; ++i) acc[q][e][i] = fmaf(as[i], f[e], acc[q][e][i]);
                } else {
                  float w[E];
                  decode_w<WT>(raw[k][q], w);
#pragma unroll
                  for (int e = 0; e < E; ++e)
#pragma unroll
                    for (int i = 0; i < NB; ++i) acc[q][e][i] = fmaf(av[i], w[e], acc[q][e][i]);
                }
              }
            }
          }
        }
      }
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < UPT; ++q)
#pragma unroll
      for (int e = 0; e < E; ++e)
#pragma unroll
        for (int i = 0; i < NB; ++i)
          red[((size_t)warp * V + (q * E + e) * NB + i) * 32 + lane] = WT == kQ4_0 ? acc[q][e][i] - corr[i] : acc[q][e][i];
    __syncthreads();
    for (int x = threadIdx.x; x < V * 32; x += blockDim.x) {
      const int ln = x & 31, y = x >> 5;
      const int i = y % NB, q = (y / NB) / E, e = (y / NB) % E;
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kDnWarps; ++w) sum += red[((size_t)w * V + y) * 32 + ln];
      const int un = c * 32 * UPT + ln + 32 * q;
      if (un < units && i < nb) partial[((int64_t)r * B + b0 + i) * d + unit_col<WT>(un, e)] = sum;
    }
  }
}

// ---------------------------------------------------------------------------
// Split-K reduction: y = b2 + sum_g partial[g] in a fixed order.  A CTA covers
// 32 float4 columns x 8 partial groups; group k sums partials g = k mod 8 in
// ascending order, then the 8 group sums are added in order.
__global__ void __launch_bounds__(256) k_ffn_reduce(const float* partial, int G, int BD,
                                                    const float* __restrict__ b2, int d, float* __restrict__ y) {
  __shared__ float4 grp[8][32];
  pdl_trigger();
  pdl_wait();
  const int col4 = blockIdx.x * 32 + (threadIdx.x & 31);
  const int k = threadIdx.x >> 5;
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  if (col4 * 4 < BD) {
    for (int g = k; g < G; g += 8) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(partial + (int64_t)g * BD) + col4);
      s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
    }
  }
  grp[k][threadIdx.x & 31] = s;
  __syncthreads();
  if (k == 0 && col4 * 4 < BD) {
    float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
    if (b2) {
      const int e = (col4 * 4) % d;
      t = *reinterpret_cast<const float4*>(b2 + e);
    }
    for (int q = 0; q < 8; ++q) {
      const float4 v = grp[q][threadIdx.x];
      t.x += v.x; t.y += v.y; t.z += v.z; t.w += v.w;
    }
    reinterpret_cast<float4*>(y)[col4] = t;
  }
}

// ---------------------------------------------------------------------------
// Stack glue: x = h + y; h_out = x * rsqrt(mean(x^2) + eps).  One CTA per
// token; each thread keeps up to kNormUnits 8-element units of x in registers
// (16-byte loads and stores), so h and y are read once.
constexpr int kNormUnits = 2;

template <int HT>
__global__ void __launch_bounds__(1024) k_rmsnorm(const void* h, const float* y, int d,
                                                  float eps, void* __restrict__ h_out) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x;
  __shared__ float red[32];
  const int units = d / 8;
  float x[kNormUnits][8];
  float ss = 0.f;
#pragma unroll
  for (int v = 0; v < kNormUnits; ++v) {
    const int u = threadIdx.x + v * blockDim.x;
    if (u < units) {
      const int64_t e0 = (int64_t)b * d + 8 * u;
      const float4 y0 = __ldcg(reinterpret_cast<const float4*>(y + e0));
      const float4 y1 = __ldcg(reinterpret_cast<const float4*>(y + e0) + 1);
      float hv[8];
      if constexpr (HT == kF32) {
        const float4 a = __ldcg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(h) + e0));
        const float4 c = __ldcg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(h) + e0) + 1);
        hv[0] = a.x; hv[1] = a.y; hv[2] = a.z; hv[3] = a.w; hv[4] = c.x; hv[5] = c.y; hv[6] = c.z; hv[7] = c.w;
      } else {
        const uint4 q = __ldcg(reinterpret_cast<const uint4*>(reinterpret_cast<const __half*>(h) + e0));
        float2 f;
        f = h2f2(q.x); hv[0] = f.x; hv[1] = f.y;
        f = h2f2(q.y); hv[2] = f.x; hv[3] = f.y;
        f = h2f2(q.z); hv[4] = f.x; hv[5] = f.y;
        f = h2f2(q.w); hv[6] = f.x; hv[7] = f.y;
      }
      const float yv[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        x[v][e] = hv[e] + yv[e];
        ss = fmaf(x[v][e], x[v][e], ss);
      }
    }
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += red[w];
  const float inv = rsqrtf(tot / (float)d + eps);
#pragma unroll
  for (int v = 0; v < kNormUnits; ++v) {
    const int u = threadIdx.x + v * blockDim.x;
    if (u < units) {
      const int64_t e0 = (int64_t)b * d + 8 * u;
      if constexpr (HT == kF32) {
        float* o = reinterpret_cast<float*>(h_out) + e0;
        reinterpret_cast<float4*>(o)[0] = make_float4(x[v][0] * inv, x[v][1] * inv, x[v][2] * inv, x[v][3] * inv);
        reinterpret_cast<float4*>(o)[1] = make_float4(x[v][4] * inv, x[v][5] * inv, x[v][6] * inv, x[v][7] * inv);
      } else {
        uint4 q;
        __half2 t;
        t = __floats2half2_rn(x[v][0] * inv, x[v][1] * inv); q.x = *reinterpret_cast<uint32_t*>(&t);
        t = __floats2half2_rn(x[v][2] * inv, x[v][3] * inv); q.y = *reinterpret_cast<uint32_t*>(&t);
        t = __floats2half2_rn(x[v][4] * inv, x[v][5] * inv); q.z = *reinterpret_cast<uint32_t*>(&t);
        t = __floats2half2_rn(x[v][6] * inv, x[v][7] * inv); q.w = *reinterpret_cast<uint32_t*>(&t);
        *reinterpret_cast<uint4*>(reinterpret_cast<__half*>(h_out) + e0) = q;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Launchers (dtype dispatch).

constexpr int kNB = 4;  // tokens per pass in the CUDA-core kernels

cudaError_t launch_pred_u(int ptype, const void* P1, const void* P1_sc, const void* h, int B, int d, int r, float* u,
                          int sms, cudaStream_t st) {
  const int grid = min((r + 7) / 8, sms * 8);
  if (ptype == kF32) k_pred_u<kF32, kNB><<<grid, 256, 0, st>>>(P1, nullptr, h, B, d, r, u);
  else if (ptype == kF16) k_pred_u<kF16, kNB><<<grid, 256, 0, st>>>(P1, nullptr, h, B, d, r, u);
  else k_pred_u<kQ4_0, kNB><<<grid, 256, 0, st>>>(P1, P1_sc, h, B, d, r, u);
  return cudaGetLastError();
}

cudaError_t launch_pred_score(int ptype, const void* P2, const void* P2_sc, const float* bp, const float* u, int B,
                              int r, int C, float thr, uint32_t* tile_mask, int* tile_count, cudaStream_t st) {
  const int tiles = (C + 255) / 256;
  if (tiles == 0) return cudaSuccess;
  if (ptype == kF32)
    k_pred_score<kF32, kNB><<<tiles, 256, 0, st>>>(P2, nullptr, bp, u, B, r, C, thr, tile_mask, tile_count);
  else if (ptype == kF16)
    k_pred_score<kF16, kNB><<<tiles, 256, 0, st>>>(P2, nullptr, bp, u, B, r, C, thr, tile_mask, tile_count);
  else
    k_pred_score<kQ4_0, kNB><<<tiles, 256, 0, st>>>(P2, P2_sc, bp, u, B, r, C, thr, tile_mask, tile_count);
  return cudaGetLastError();
}

cudaError_t launch_compact(const uint32_t* tile_mask, const int* tile_count, int C, int n_hot, int32_t* idx,
                           int32_t* count, cudaStream_t st) {
  const int tiles = (C + 255) / 256;
  if (tiles == 0) return cudaMemsetAsync(count, 0, sizeof(int32_t), st);
  const cudaError_t e = launch_pdl(k_compact, dim3(tiles), dim3(256), 0, st, tile_mask, tile_count, tiles, n_hot, idx, count);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int WT, int HT>
static void act_dispatch(int act, int grid, cudaStream_t st, const void* h, int B, int d, int ffn, int n_hot,
                         const int32_t* idx, const int32_t* count, const void* wg, const void* wg_sc, const void* wu,
                         const void* wu_sc, const float* b1, float* a, int n_max, int* status) {
  if (act == kReglu)
    k_ffn_act<WT, HT, kReglu, kNB><<<grid, 256, 0, st>>>(h, B, d, ffn, n_hot, idx, count, wg, wg_sc, wu, wu_sc, b1,
                                                         a, n_max, status);
  else if (act == kRelu2)
    k_ffn_act<WT, HT, kRelu2, kNB><<<grid, 256, 0, st>>>(h, B, d, ffn, n_hot, idx, count, wg, wg_sc, wu, wu_sc, b1,
                                                         a, n_max, status);
  else
    k_ffn_act<WT, HT, kRelu, kNB><<<grid, 256, 0, st>>>(h, B, d, ffn, n_hot, idx, count, wg, wg_sc, wu, wu_sc, b1,
                                                        a, n_max, status);
}

cudaError_t launch_ffn_act(int wtype, int htype, int act, const void* h, int B, int d, int ffn, int n_hot,
                           const int32_t* idx, const int32_t* count, const void* wg, const void* wg_sc,
                           const void* wu, const void* wu_sc, const float* b1, float* a, int n_max, int* status,
                           int sms, cudaStream_t st) {
  const int grid = sms * 8;
  if (htype == kF32) {
    if (wtype == kF32) act_dispatch<kF32, kF32>(act, grid, st, h, B, d, ffn, n_hot, idx, count, wg, wg_sc, wu, wu_sc, b1, a, n_max, status);
    else if (wtype == kF16) act_dispatch<kF16, kF32>(act, grid, st, h, B, d, ffn, n_hot, idx, count, wg, wg_sc, wu, wu_sc, b1, a, n_max, status);
    else act_dispatch<kQ4_0, kF32>(act, grid, st, h, B, d, ffn, n_hot, idx, count, wg, wg_sc, wu, wu_sc, b1, a, n_max, status);
  } else {
    if (wtype == kF32) act_dispatch<kF32, kF16>(act, grid, st, h, B, d, ffn, n_hot, idx, count, wg, wg_sc, wu, wu_sc, b1, a, n_max, status);
    else if (wtype == kF16) act_dispatch<kF16, kF16>(act, grid, st, h, B, d, ffn, n_hot, idx, count, wg, wg_sc, wu, wu_sc, b1, a, n_max, status);
    else act_dispatch<kQ4_0, kF16>(act, grid, st, h, B, d, ffn, n_hot, idx, count, wg, wg_sc, wu, wu_sc, b1, a, n_max, status);
  }
  return cudaGetLastError();
}

int down_ranges(int d, int sms) {
  const int chunks = (d + 511) / 512;
  const int R = (3 * sms) / chunks;
  return R < 1 ? 1 : (R > kGMax ? kGMax : R);
}

cudaError_t launch_ffn_down(int wtype, int B, int d, int ffn, int n_hot, const int32_t* idx, const int32_t* count,
                            const void* wd, const void* wd_sc, const float* a, int n_max, float* partial, int G,
                            cudaStream_t st, const float* pre, int pre_S, int pre_R, const float* b1, int act) {
  if (G < 1 || G > kGMax) return cudaErrorInvalidValue;
  const dim3 grid((d + 511) / 512, G);
  const size_t smem = (size_t)kDnWarps * 16 * kNB * 32 * sizeof(float);
  static_assert((size_t)kDnWarps * 16 * kNB * 32 >= (size_t)(1 + kNB) * kDnCap, "the staging fits the reduction buffer");
  cudaError_t e;
  if (wtype == kF32) {
    if ((e = cudaFuncSetAttribute(k_ffn_down<kF32, kNB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
      return e;
    k_ffn_down<kF32, kNB><<<grid, kDnWarps * 32, smem, st>>>(B, d, ffn, n_hot, idx, count, wd, wd_sc, a, n_max, partial, pre, pre_S, pre_R, b1, act);
  } else if (wtype == kF16) {
    if ((e = cudaFuncSetAttribute(k_ffn_down<kF16, kNB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
      return e;
    k_ffn_down<kF16, kNB><<<grid, kDnWarps * 32, smem, st>>>(B, d, ffn, n_hot, idx, count, wd, wd_sc, a, n_max, partial, pre, pre_S, pre_R, b1, act);
  } else {
    if ((e = cudaFuncSetAttribute(k_ffn_down<kQ4_0, kNB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
      return e;
    k_ffn_down<kQ4_0, kNB><<<grid, kDnWarps * 32, smem, st>>>(B, d, ffn, n_hot, idx, count, wd, wd_sc, a, n_max,
                                                              partial, pre, pre_S, pre_R, b1, act);
  }
  return cudaGetLastError();
}

cudaError_t launch_ffn_reduce(const float* partial, int G, int B, int d, const float* b2, float* y, cudaStream_t st) {
  const int BD = B * d;
  const int grid = (BD / 4 + 31) / 32;
  const cudaError_t e = launch_pdl(k_ffn_reduce, dim3(grid), dim3(256), 0, st, partial, G, BD, b2, d, y);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_rmsnorm(int htype, const void* h, const float* y, int B, int d, float eps, void* h_out,
                           cudaStream_t st) {
  // one CTA per token, one thread per 8-element unit (at most kNormUnits units per thread)
  const int units = d / 8;
  int threads = (units + kNormUnits - 1) / kNormUnits;
  threads = (threads + 31) / 32 * 32;
  if (threads > 1024 || d % 8 != 0) return cudaErrorInvalidValue;
  const cudaError_t e = htype == kF32 ? launch_pdl(k_rmsnorm<kF32>, dim3(B), dim3(threads), 0, st, h, y, d, eps, h_out)
                                      : launch_pdl(k_rmsnorm<kF16>, dim3(B), dim3(threads), 0, st, h, y, d, eps, h_out);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace pi
