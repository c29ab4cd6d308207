// pi_stack.cu -- one persistent, cooperative kernel for a whole decode step
// through every layer of the stack (token blocks of 1 or 2).
//
// Pages: unite.ai "PowerInfer: Tüketici Düzeyinde bir GPU ile Hızlı Büyük Dil
// Modeli Sunucusu" -- "Adaptif Sparsite Predictor’ları" (a per-layer predictor
// picks the active neurons), "Nöron Bilinçli Operatör" (operators on single
// rows of the up/gate matrices and single columns of the down matrix),
// "Nöron Yerleştirme ve Yönetimi" (hot neurons stored first, with a table back
// to the original rows); GeekNews "Serving model bahasa besar ...",
// "Metode inferensi hibrida CPU/GPU" (the always-active block runs densely on
// the GPU) and "Keterbatasan dan FAQ" (ReLU, ReGLU, squared ReLU).
//
// Design (one CTA per SM, G CTAs, grid-wide barriers are bounded spins):
//   * a producer warp streams every byte the CTA needs into a shared-memory
//     byte ring with 1-D bulk copies (cp.async.bulk, mbarrier completion), in
//     a fixed order per layer: its P1 rows, its block of P2 rows, its share
//     of the hot neurons (gate/up/down rows of each neuron as one item), then
//     -- once every CTA has scored its P2 rows -- its share of the predicted
//     cold neurons.  Nothing but the cold rows depends on the predictor, so
//     the ring keeps HBM busy across the grid barriers.
//   * consumer warps own 16 fixed columns of d per thread: the token block
//     and the fp32 partial output stay in registers for the whole layer.
//   * per layer: P1 rows -> u (global) -> barrier U -> P2 scores of the CTA's
//     cold rows -> local ascending list + count -> barrier S -> hot neurons ->
//     cold share of the global list -> partial y reduced into an fp32
//     accumulator with vector atomics -> barrier Y -> residual + RMSNorm glue
//     computed redundantly by every CTA -> next layer.
//   * the cold list is ordered: CTA c's active rows are ascending and precede
//     CTA c+1's, so the concatenation is the ascending list pi_predict writes.
#include <cuda_runtime.h>
#include <stdint.h>

#include "pi_common.cuh"
#include "pi_mma.cuh"
#include "pi_stack.cuh"
#include "pi_sync.cuh"

namespace pi {

namespace {

// ----------------------------------------------------------------------------
// column ownership: consumer thread t of T owns 16 columns of d, as NRUN runs
// of RUN consecutive columns whose layout follows the weight type.

template <int WT, int EPT>
struct Own {
  static_assert(EPT == 8 || EPT == 16, "8 or 16 columns per thread");
  static constexpr int RUN = (WT == kF32) ? 4 : (WT == kQ4_0 ? EPT / 2 : 8);
  static constexpr int NRUN = EPT / RUN;
  __device__ __forceinline__ static int col(int t, int T, int k) {
    if constexpr (WT == kQ4_0) {
      // EPT/2 bytes of one Q4_0 block: low nibbles give a run, high nibbles the run 16 columns on
      constexpr int PER_BLK = 32 / EPT;  // threads per 32-column block
      return (t / PER_BLK) * 32 + (t % PER_BLK) * (EPT / 2) + k * 16;
    } else {
      return (t + k * T) * RUN;
    }
  }
};

// 16 owned values of a d-row of element type X (kF32/kF16) at `row` (shared or global).
template <int WT, int EPT, int X>
__device__ __forceinline__ void row_vals(const uint8_t* row, int t, int T, float (&v)[EPT]) {
  using O = Own<WT, EPT>;
#pragma unroll
  for (int k = 0; k < O::NRUN; ++k) {
    const int c = O::col(t, T, k);
    float* o = v + k * O::RUN;
    if constexpr (X == kF16) {
      if constexpr (O::RUN == 8) {
        const uint4 q = *reinterpret_cast<const uint4*>(row + 2 * c);
        float2 f;
        f = h2f2(q.x); o[0] = f.x; o[1] = f.y;
        f = h2f2(q.y); o[2] = f.x; o[3] = f.y;
        f = h2f2(q.z); o[4] = f.x; o[5] = f.y;
        f = h2f2(q.w); o[6] = f.x; o[7] = f.y;
      } else {
        const uint2 q = *reinterpret_cast<const uint2*>(row + 2 * c);
        float2 f;
        f = h2f2(q.x); o[0] = f.x; o[1] = f.y;
        f = h2f2(q.y); o[2] = f.x; o[3] = f.y;
      }
    } else {
#pragma unroll
      for (int e = 0; e < O::RUN; e += 4) {
        const float4 q = *reinterpret_cast<const float4*>(row + 4 * (c + e));
        o[e] = q.x; o[e + 1] = q.y; o[e + 2] = q.z; o[e + 3] = q.w;
      }
    }
  }
}

// EPT owned values of a Q4_0 row laid out as [qs d/2 bytes][sc d/16 bytes]:
// EPT/2 consecutive qs bytes of one block; their low nibbles are the first
// run, their high nibbles the run 16 columns on; x = s * (q - 8).
template <int EPT>
__device__ __forceinline__ void q4_vals(const uint8_t* row, int d, int t, float (&v)[EPT]) {
  constexpr int NB = EPT / 2;         // qs bytes per thread
  constexpr int PER_BLK = 32 / EPT;   // threads per block
  uint32_t q[NB / 4];
  if constexpr (NB == 8) {
    const uint2 qq = *reinterpret_cast<const uint2*>(row + NB * t);
    q[0] = qq.x;
    q[1] = qq.y;
  } else {
    q[0] = *reinterpret_cast<const uint32_t*>(row + NB * t);
  }
  const uint16_t sb = *reinterpret_cast<const uint16_t*>(row + d / 2 + 2 * (t / PER_BLK));
  const float s = half_bits_to_float(sb);
#pragma unroll
  for (int w = 0; w < NB / 4; ++w)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t b = (q[w] >> (8 * k)) & 0xffu;
      v[w * 4 + k] = s * (float)((int)(b & 15u) - 8);
      v[NB + w * 4 + k] = s * (float)((int)(b >> 4) - 8);
    }
}

template <int WT, int EPT>
__device__ __forceinline__ void w_vals(const uint8_t* row, int d, int t, int T, float (&v)[EPT]) {
  if constexpr (WT == kQ4_0) q4_vals<EPT>(row, d, t, v);
  else row_vals<WT, EPT, WT>(row, t, T, v);
}

template <int WT, int EPT, int X>
__device__ __forceinline__ void store_vals(uint8_t* row, int t, int T, const float (&v)[EPT]) {
  using O = Own<WT, EPT>;
#pragma unroll
  for (int k = 0; k < O::NRUN; ++k) {
    const int c = O::col(t, T, k);
    const float* o = v + k * O::RUN;
    if constexpr (X == kF16) {
#pragma unroll
      for (int e = 0; e < O::RUN; e += 2) {
        *reinterpret_cast<__half2*>(row + 2 * (c + e)) = __floats2half2_rn(o[e], o[e + 1]);
      }
    } else {
#pragma unroll
      for (int e = 0; e < O::RUN; e += 4) {
        *reinterpret_cast<float4*>(row + 4 * (c + e)) = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
      }
    }
  }
}

__device__ __forceinline__ float round_to(int X, float v) {
  return X == kF16 ? __half2float(__float2half_rn(v)) : v;
}

__device__ __forceinline__ float act_eval(int act, float g, float v) {
  if (act == kReglu) return fmaxf(g, 0.f) * v;
  const float r = fmaxf(g, 0.f);
  return act == kRelu2 ? r * r : r;
}

__device__ __forceinline__ int wrow_bytes(int WT_, int d) {
  return WT_ == kQ4_0 ? d / 2 + d / 16 : d * (WT_ == kF16 ? 2 : 4);
}

struct Smem {
  uint8_t* ring;
  uint64_t* full;
  uint64_t* empty;
  uint64_t* list_bar;
  uint32_t* item_off;
  uint32_t* istart;  // producer-private: start/size of the items in flight
  float* u;          // [B][r] split layout (see load_u)
  float* bp;
  float* b1hot;
  int* cidx;
  float* cb1;
  uint8_t* act;
  float* red;        // [2][NW][2B]
  int* prefix;       // [G + 1]
  int* misc;         // [0] cold_n, [1] gen_start
  uint8_t* hb;       // [B][d + 8] fp16 token rows (tensor-core operand)
  uint8_t* ub;       // [2B][r + 8] fp16 u rows: hi and lo parts of each token's u
  uint8_t* zero;     // 16 zero bytes (operand rows beyond the token count)
  float* redp;       // [NW][16][2] P1 partial dots
};

__device__ __forceinline__ Smem carve(uint8_t* base, const StackParams& p) {
  Smem s;
  s.ring = base;
  s.full = reinterpret_cast<uint64_t*>(base + p.off_bars);
  s.empty = s.full + kNQ;
  s.list_bar = s.empty + kNQ;
  s.item_off = reinterpret_cast<uint32_t*>(base + p.off_itemoff);
  s.istart = s.item_off + kNQ;
  s.u = reinterpret_cast<float*>(base + p.off_u);
  s.bp = reinterpret_cast<float*>(base + p.off_bp);
  s.b1hot = reinterpret_cast<float*>(base + p.off_b1hot);
  s.cidx = reinterpret_cast<int*>(base + p.off_cidx);
  s.cb1 = reinterpret_cast<float*>(base + p.off_cb1);
  s.act = base + p.off_act;
  s.red = reinterpret_cast<float*>(base + p.off_red);
  s.prefix = reinterpret_cast<int*>(base + p.off_prefix);
  s.misc = reinterpret_cast<int*>(base + p.off_misc);
  s.hb = base + p.off_hb;
  s.ub = base + p.off_ub;
  s.zero = base + p.off_zero;
  s.redp = reinterpret_cast<float*>(base + p.off_redp);
  return s;
}

__device__ __forceinline__ int share_lo(int n, int c, int G) { return (int)((int64_t)n * c / G); }

// CTA-wide (consumer warps) sum of NV values per thread; every thread gets the
// same totals (same butterfly order in every warp).  The two scratch buffers alternate
// (stride MAXV per warp) so that the next call's writes cannot overtake this
// call's reads.  Returns the OR of `flag` over the consumer threads.
template <int NV, int MAXV>
__device__ __forceinline__ bool cta_reduce(float (&v)[NV], float* red_base, int& par, int warp, int lane, int NW,
                                           int T, bool flag) {
#pragma unroll
  for (int i = 0; i < NV; ++i) v[i] = warp_sum(v[i]);
  float* red = red_base + par * (kMaxConsumers / 32) * MAXV;
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < NV; ++i) red[warp * MAXV + i] = v[i];
  }
  flag = named_sync_or(1, T, flag);
  // lane w reads warp w's partial; a butterfly gives every lane the total
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    float a = lane < NW ? red[lane * MAXV + i] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    v[i] = a;
  }
  par ^= 1;
  return flag;
}

// ----------------------------------------------------------------------------
// producer (one warp; lane 0 issues the copies)

struct Producer {
  const StackParams& p;
  Smem& s;
  Ctrl* ctrl;
  uint32_t item = 0;  // next item index
  uint32_t rel = 0;   // items known consumed
  uint32_t head = 0;  // next free ring byte

  __device__ Producer(const StackParams& p_, Smem& s_) : p(p_), s(s_), ctrl(p_.ctrl) {}

  __device__ bool wait_consumed() {
    const uint32_t q = rel % kNQ;
    if (!mbar_wait(&s.empty[q], (rel / kNQ) & 1u, ctrl)) return false;
    ++rel;
    return true;
  }

  // Reserve `bytes` contiguous ring bytes for the next item; returns the offset.
  __device__ bool alloc(uint32_t bytes, uint32_t& pos) {
    const uint32_t R = (uint32_t)p.ring_bytes;
    for (;;) {
      if (item - rel >= (uint32_t)kNQ) {
        if (!wait_consumed()) return false;
        continue;
      }
      if (rel == item) {  // ring empty
        pos = (head + bytes <= R) ? head : 0;
        return true;
      }
      const uint32_t tail = s.istart[rel % kNQ];
      if (head > tail) {
        if (head + bytes <= R) { pos = head; return true; }
        if (bytes <= tail) { pos = 0; return true; }
      } else if (head + bytes <= tail) {
        pos = head;
        return true;
      }
      if (!wait_consumed()) return false;
    }
  }

  // One item of `nrows` rows of `row_bytes` each: row i comes from
  // src + i * src_stride and lands at dst_stride * i past a 128-byte aligned
  // start shifted by `skew` bytes (skew and padding keep ldmatrix rows of
  // consecutive rows/items on different shared-memory banks).
  __device__ bool issue_rows(const uint8_t* src, int64_t src_stride, int nrows, uint32_t row_bytes,
                             uint32_t dst_stride, uint32_t skew) {
    const uint32_t total = nrows * dst_stride + 128 + skew;
    uint32_t pos;
    if (!alloc(total, pos)) return false;
    const uint32_t start = ((pos + 127u) & ~127u) + skew;
    const uint32_t q = item % kNQ;
    s.item_off[q] = start;
    s.istart[q] = pos;
    mbar_arrive_expect_tx(&s.full[q], nrows * row_bytes);
    for (int i = 0; i < nrows; ++i) bulk_g2s(s.ring + start + i * dst_stride, src + i * src_stride, row_bytes, &s.full[q]);
    head = pos + total;
    ++item;
    return true;
  }

  // One item made of up to 6 contiguous source segments, copied back to back.
  __device__ bool issue(int nseg, const void* const* src, const uint32_t* bytes) {
    uint32_t total = 0;
    for (int i = 0; i < nseg; ++i) total += bytes[i];
    uint32_t pos;
    if (!alloc(total, pos)) return false;
    const uint32_t q = item % kNQ;
    s.item_off[q] = pos;
    s.istart[q] = pos;
    mbar_arrive_expect_tx(&s.full[q], total);
    uint32_t o = pos;
    for (int i = 0; i < nseg; ++i) {
      bulk_g2s(s.ring + o, src[i], bytes[i], &s.full[q]);
      o += bytes[i];
    }
    head = pos + total;
    ++item;
    return true;
  }

  // One neuron: its gate (ReGLU only), up and down rows.  Row m of the item
  // starts m * (wrb + 16) bytes past a 128-byte aligned base that is shifted
  // by 32 * (neuron sequence number mod 4) bytes, so that the gate and up
  // rows of four consecutive neurons fall on eight different shared-memory
  // bank groups (conflict-free ldmatrix).  Q4_0 rows hold qs then sc.
  uint32_t nseq = 0;
  __device__ bool issue_neuron(const StackLayer& Ly, int j, int wt, int gated) {
    const int d = p.d;
    const uint32_t wrb = wt == kQ4_0 ? (uint32_t)(d / 2 + d / 16) : (uint32_t)(d * (wt == kF16 ? 2 : 4));
    const uint32_t wrp = wrb + 16;
    const int nrow = gated ? 3 : 2;
    const uint32_t skew = 32u * (nseq & 3u);
    ++nseq;
    const uint32_t total = nrow * wrp + 128 + skew;
    uint32_t pos;
    if (!alloc(total, pos)) return false;
    const uint32_t start = ((pos + 127u) & ~127u) + skew;
    const uint32_t q = item % kNQ;
    s.item_off[q] = start;
    s.istart[q] = pos;
    mbar_arrive_expect_tx(&s.full[q], nrow * wrb);
    const void* rows[3];
    const void* scs[3];
    int m = 0;
    if (gated) { rows[m] = Ly.wg; scs[m++] = Ly.wg_sc; }
    rows[m] = Ly.wu; scs[m++] = Ly.wu_sc;
    rows[m] = Ly.wd; scs[m++] = Ly.wd_sc;
    for (int i = 0; i < nrow; ++i) {
      uint8_t* dst = s.ring + start + i * wrp;
      if (wt == kQ4_0) {
        bulk_g2s(dst, reinterpret_cast<const uint8_t*>(rows[i]) + (int64_t)j * (d / 2), d / 2, &s.full[q]);
        bulk_g2s(dst + d / 2, reinterpret_cast<const uint8_t*>(scs[i]) + (int64_t)j * (d / 16), d / 16, &s.full[q]);
      } else {
        bulk_g2s(dst, reinterpret_cast<const uint8_t*>(rows[i]) + (int64_t)j * wrb, wrb, &s.full[q]);
      }
    }
    head = pos + total;
    ++item;
    return true;
  }

  // Drain: wait for every issued copy to land before the CTA may exit.
  __device__ void drain() {
    for (uint32_t i = rel; i < item; ++i) mbar_wait(&s.full[i % kNQ], (i / kNQ) & 1u, ctrl);
  }
};

// ----------------------------------------------------------------------------

template <int WT, int PT, int B, int EPT>
__global__ void __launch_bounds__(kMaxConsumers + 32, 1) k_stack(const __grid_constant__ StackParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem s = carve(smem_raw, p);
  Ctrl* ctrl = p.ctrl;
  const int G = gridDim.x, c = blockIdx.x;
  const int T = p.T, NW = T / 32;
  const int d = p.d, r = p.rank, H = p.n_hot, C = p.ffn - p.n_hot;
  const int gated = p.act == kReglu;
  const int ep = PT == kF16 ? 2 : 4;
  constexpr int K = kYCopies;

  if (threadIdx.x == 0) {
    for (int q = 0; q < kNQ; ++q) {
      mbar_init(&s.full[q], 1);
      mbar_init(&s.empty[q], NW);
      s.item_off[q] = 0u;  // in-ring offsets even before the first item of a slot
      s.istart[q] = 0u;
    }
    mbar_init(s.list_bar, 1);
    mbar_fence_init();
    s.misc[1] = (int)ld_acquire_u32(&ctrl->bar_base);
  }
  __syncthreads();
  const unsigned base = (unsigned)s.misc[1];

  // shares that do not depend on the predictor
  const int k0 = share_lo(r, c, G), k1 = share_lo(r, c + 1, G);
  const int c0 = share_lo(C, c, G), c1 = share_lo(C, c + 1, G);
  const int j0 = share_lo(H, c, G), j1 = share_lo(H, c + 1, G);

  if (threadIdx.x < 32) {
    // ======================= producer warp =======================
    const int lane = threadIdx.x;
    Producer pr(p, s);
    bool ok = true;
    for (int l = 0; l < p.L && ok; ++l) {
      const StackLayer& Ly = p.layers[l];
      if (lane == 0) {
        if constexpr (PT == kF16) {
          // tensor-core predictor: skewed P1 rows, P2 in 16-row tiles with padded rows
          for (int k = k0; k < k1 && ok; ++k)
            ok = pr.issue_rows(reinterpret_cast<const uint8_t*>(Ly.P1) + (int64_t)k * d * 2, 0, 1, d * 2, d * 2,
                               16u * (uint32_t)((k - k0) & 7));
          for (int cc = c0; cc < c1 && ok; cc += 16)
            ok = pr.issue_rows(reinterpret_cast<const uint8_t*>(Ly.P2) + (int64_t)cc * r * 2, (int64_t)r * 2,
                               min(16, c1 - cc), r * 2, r * 2 + 16, 0);
        } else {
          for (int k = k0; k < k1 && ok; ++k) {
            const void* src = reinterpret_cast<const uint8_t*>(Ly.P1) + (int64_t)k * d * ep;
            const uint32_t by = d * ep;
            ok = pr.issue(1, &src, &by);
          }
          for (int cc = c0; cc < c1 && ok; cc += NW) {
            const int rows = min(NW, c1 - cc);
            const void* src = reinterpret_cast<const uint8_t*>(Ly.P2) + (int64_t)cc * r * ep;
            const uint32_t by = rows * r * ep;
            ok = pr.issue(1, &src, &by);
          }
        }
        for (int j = j0; j < j1 && ok; ++j) ok = pr.issue_neuron(Ly, j, WT, gated);
        // the cold rows need every CTA's scores: barrier S of this layer
        if (ok) ok = grid_wait(ctrl, base, 3 * l + 1, G);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      __syncwarp();
      if (!ok) break;
      // prefix over the per-CTA counts (all loads in flight at once)
      constexpr int kMaxChunks = (kGMaxCtas + 31) / 32;
      int cv[kMaxChunks];
#pragma unroll 1
      for (int m = 0; m < kMaxChunks; ++m) {
        const int i = m * 32 + lane;
        cv[m] = i < G ? __ldcg(p.seg_cnt + i) : 0;
      }
      if (lane == 0) s.prefix[0] = 0;
      int run = 0;
#pragma unroll 1
      for (int m = 0; m < kMaxChunks; ++m) {
        int x = cv[m];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        const int i = m * 32 + lane;
        if (i < G) s.prefix[i + 1] = run + x;
        run += __shfl_sync(0xffffffffu, x, 31);
      }
      __syncwarp();
      const int A = run;
      const int q0 = share_lo(A, c, G), q1 = share_lo(A, c + 1, G);
      for (int q = q0 + lane; q < q1; q += 32) {
        int lo = 0, hi = G;  // last CTA with prefix[cta] <= q
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if (s.prefix[mid] <= q) lo = mid;
          else hi = mid;
        }
        s.cidx[q - q0] = __ldcg(p.seg + (int64_t)lo * p.seg_cap + (q - s.prefix[lo]));
      }
      if (lane == 0) s.misc[0] = q1 - q0;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(s.list_bar);
        for (int q = 0; q < q1 - q0 && ok; ++q) ok = pr.issue_neuron(Ly, s.cidx[q], WT, gated);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      // outputs (off the critical path): this CTA's part of the ascending list, and the count
      const int my_n = s.prefix[c + 1] - s.prefix[c];
      for (int i = lane; i < my_n; i += 32)
        p.idx[(int64_t)l * C + s.prefix[c] + i] = __ldcg(p.seg + (int64_t)c * p.seg_cap + i);
      if (c == 0 && lane == 0) p.counts[l] = A;
      __syncwarp();
    }
    if (lane == 0) pr.drain();
    return;
  }

  // ======================= consumer warps =======================
  const int t = threadIdx.x - 32;
  const int warp = t >> 5, lane = t & 31;
  uint32_t witem = 0, ritem = 0;  // next item to wait for / to release
  int par = 0;
  float h[B][EPT], y[B][EPT];

  auto wait_item = [&](uint32_t& off) -> bool {
    const uint32_t q = witem % kNQ;
    const bool okw = mbar_wait(&s.full[q], (witem / kNQ) & 1u, ctrl);
    off = okw ? s.item_off[q] : 0u;  // after a timeout, reads stay inside the ring
    ++witem;
    return okw;
  };
  auto release_item = [&]() {
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[ritem % kNQ]);
    ++ritem;
  };

  // layer-0 input
#pragma unroll
  for (int b = 0; b < B; ++b)
    row_vals<WT, EPT, PT>(reinterpret_cast<const uint8_t*>(p.h_in) + (int64_t)b * d * ep, t, T, h[b]);
  if (c == 0 && p.h_trace) {
#pragma unroll
    for (int b = 0; b < B; ++b) store_vals<WT, EPT, PT>(reinterpret_cast<uint8_t*>(p.h_trace) + (int64_t)b * d * ep, t, T, h[b]);
  }
  const int HS = 2 * d + 16;  // byte stride of the fp16 token rows in shared memory
  const int US = 2 * r + 16;  // byte stride of the fp16 u rows
  if constexpr (PT == kF16) {
#pragma unroll
    for (int b = 0; b < B; ++b) store_vals<WT, EPT, kF16>(s.hb + b * HS, t, T, h[b]);
    if (t < 4) reinterpret_cast<uint32_t*>(s.zero)[t] = 0u;
  }
  const int ybuf4 = K * B * d / 4;  // float4s per accumulator buffer (K copies)
  {
    const int z0 = share_lo(ybuf4, c, G), z1 = share_lo(ybuf4, c + 1, G);
    for (int i = z0 + t; i < z1; i += T) reinterpret_cast<float4*>(p.yacc)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }

  for (int l = 0; l < p.L; ++l) {
    const StackLayer& Ly = p.layers[l];
    // small per-layer vectors of this CTA's shares: loaded now, stored to
    // shared memory after the P1 rows so that the load latency is hidden
    float bp_v[kShareRegs], b1_v[kShareRegs];
#pragma unroll
    for (int i = 0; i < kShareRegs; ++i) {
      const int x = t + i * T;
      bp_v[i] = (Ly.bp && x < c1 - c0) ? __ldg(Ly.bp + c0 + x) : 0.f;
      b1_v[i] = (Ly.b1 && x < j1 - j0) ? __ldg(Ly.b1 + j0 + x) : 0.f;
    }

    // ---- predictor step 1: u = ReLU(P1 h) ----
    bool to = false;
    if constexpr (PT == kF16) {
      // Tensor cores: the CTA's (<= 16) P1 rows are the A tile, the fp16
      // token rows the B tile; warps split d, partial dots meet in shared memory.
      named_sync(1, T);  // token rows (written by the glue) are complete
      const int bn = lane & 7;
      const uint32_t b_base = (bn < B ? smem_u32(s.hb + bn * HS) + (uint32_t)(((lane >> 3) & 1) * 16) : smem_u32(s.zero));
      const uint32_t b_step = bn < B ? 32u : 0u;
      const int KS = d / 16, ks0 = warp * KS / NW, ks1 = (warp + 1) * KS / NW;
      // rows in groups of at most p.p1rows, so that a group fits in half the ring
      for (int g0 = k0; g0 < k1; g0 += p.p1rows) {
        const int nrow = min(p.p1rows, k1 - g0);
        if (g0 > k0) named_sync(1, T);  // the previous group's partial dots have been read
        for (int i = 0; i < nrow; ++i) to |= !mbar_wait(&s.full[(witem + i) % kNQ], ((witem + i) / kNQ) & 1u, ctrl);
        const int ar = lane & 15;
        const uint32_t a_base =
            smem_u32(s.ring + s.item_off[(witem + (ar < nrow ? ar : 0)) % kNQ]) + (uint32_t)((lane >> 4) * 16);
        float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
        int ks = to ? ks1 : ks0;  // no tile is read unless all its rows have landed
        for (; ks + 1 < ks1; ks += 2) {
          uint32_t a0, a1, a2, a3, b0, b1, e0, e1, e2, e3, f0, f1;
          ldsm_x4(a_base + 32u * ks, a0, a1, a2, a3);
          ldsm_x2(b_base + b_step * ks, b0, b1);
          ldsm_x4(a_base + 32u * (ks + 1), e0, e1, e2, e3);
          ldsm_x2(b_base + b_step * (ks + 1), f0, f1);
          mma_16816(acc0, a0, a1, a2, a3, b0, b1);
          mma_16816(acc1, e0, e1, e2, e3, f0, f1);
        }
        if (ks < ks1) {
          uint32_t a0, a1, a2, a3, b0, b1;
          ldsm_x4(a_base + 32u * ks, a0, a1, a2, a3);
          ldsm_x2(b_base + b_step * ks, b0, b1);
          mma_16816(acc0, a0, a1, a2, a3, b0, b1);
        }
        witem += nrow;
        for (int i = 0; i < nrow; ++i) release_item();
        // thread (g = lane/4, t4 = lane%4 == 0) holds rows g and g+8, tokens 0 and 1
        if ((lane & 3) == 0) {
          const int g = lane >> 2;
          float* rp = s.redp + warp * 32;
          rp[g * 2 + 0] = acc0[0] + acc1[0];
          rp[g * 2 + 1] = acc0[1] + acc1[1];
          rp[(g + 8) * 2 + 0] = acc0[2] + acc1[2];
          rp[(g + 8) * 2 + 1] = acc0[3] + acc1[3];
        }
        if (named_sync_or(1, T, to)) return;
        if (t < nrow * B) {
          const int row = t / B, b = t % B;
          float a = 0.f;
          for (int w = 0; w < NW; ++w) a += s.redp[w * 32 + row * 2 + b];
          p.u_g[(int64_t)b * r + g0 + row] = fmaxf(a, 0.f);
        }
      }
    } else {
    for (int kk = k0; kk < k1; kk += 4) {
      const int nrow = min(4, k1 - kk);
      float acc[4 * B];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int b = 0; b < B; ++b) acc[i * B + b] = 0.f;
        if (i < nrow) {
          uint32_t off;
          to |= !wait_item(off);
          float w[EPT];
          row_vals<WT, EPT, PT>(s.ring + off, t, T, w);
          release_item();
#pragma unroll
          for (int b = 0; b < B; ++b) {
            float a = 0.f;
#pragma unroll
            for (int e = 0; e < EPT; ++e) a = fmaf(w[e], h[b][e], a);
            acc[i * B + b] = a;
          }
        }
      }
      to = cta_reduce<4 * B, 4 * B>(acc, s.red, par, warp, lane, NW, T, to);
      if (to) return;
      if (t == 0)
        for (int i = 0; i < nrow; ++i)
          for (int b = 0; b < B; ++b) p.u_g[(int64_t)b * r + kk + i] = fmaxf(acc[i * B + b], 0.f);
    }
    }  // predictor step 1
#pragma unroll
    for (int i = 0; i < kShareRegs; ++i) {
      const int x = t + i * T;
      if (x < c1 - c0) s.bp[x] = bp_v[i];
      if (x < j1 - j0) s.b1hot[x] = b1_v[i];
    }
    named_sync(1, T);
    if (t == 0) grid_arrive(ctrl);
    {
      bool okw = true;
      if (t == 0) okw = grid_wait(ctrl, base, 3 * l, G);
      if (named_sync_or(1, T, !okw)) return;
    }
    // the other accumulator buffer is free now (its last readers passed this barrier)
    {
      float4* nxt = reinterpret_cast<float4*>(p.yacc) + (size_t)((l + 1) & 1) * ybuf4;
      const int z0 = share_lo(ybuf4, c, G), z1 = share_lo(ybuf4, c + 1, G);
      for (int i = z0 + t; i < z1; i += T) nxt[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if constexpr (PT == kF16) {
      // u -> fp16 rows for the tensor cores: row 2b = hi(u_b), row 2b+1 = lo(u_b) = u_b - hi
      for (int i = t; i < B * r; i += T) {
        const int b = i / r, k = i % r;
        const float v = __ldcg(p.u_g + i);
        const __half hi = __float2half_rn(v);
        const __half lo = __float2half_rn(v - __half2float(hi));
        reinterpret_cast<__half*>(s.ub + (2 * b) * US)[k] = hi;
        reinterpret_cast<__half*>(s.ub + (2 * b + 1) * US)[k] = lo;
      }
    } else {
      // u -> shared memory, split layout: unit m (8 values) stored as two float4
      // planes so that lane-strided reads are conflict-free.
      const int nu = r / 8;
      for (int i = t; i < B * nu; i += T) {
        const int b = i / nu, m = i % nu;
        const float4* src = reinterpret_cast<const float4*>(p.u_g + (int64_t)b * r + 8 * m);
        const float4 lo = __ldcg(src), hi = __ldcg(src + 1);
        float4* dst = reinterpret_cast<float4*>(s.u + (size_t)b * r);
        dst[m] = lo;
        dst[nu + m] = hi;
      }
    }
    named_sync(1, T);

    // ---- predictor step 2: scores of this CTA's cold rows ----
    if constexpr (PT == kF16) {
      // Tensor cores: each 16-row tile of P2 (one ring item) against the u
      // rows (hi, lo per token); warp w takes tiles w, w + NW, ...
      const int nrows = c1 - c0;
      const int ntile = (nrows + 15) / 16;
      const int bn = lane & 7;
      const uint32_t b_base = (bn < 2 * B ? smem_u32(s.ub + bn * US) + (uint32_t)(((lane >> 3) & 1) * 16) : smem_u32(s.zero));
      const uint32_t b_step = bn < 2 * B ? 32u : 0u;
      const int KS = r / 16;
      for (int it = 0; it < ntile; ++it) {
        const uint32_t myitem = witem + it;
        if (it % NW == warp) {
          to |= !mbar_wait(&s.full[myitem % kNQ], (myitem / kNQ) & 1u, ctrl);
          const int rows = min(16, nrows - 16 * it);
          const int ar = lane & 15;
          const uint32_t a_base = smem_u32(s.ring + s.item_off[myitem % kNQ]) + (uint32_t)((ar < rows ? ar : 0) * US) +
                                  (uint32_t)((lane >> 4) * 16);
          float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
          int ks = to ? KS : 0;  // the tile is read only once it has landed
          for (; ks + 1 < KS; ks += 2) {
            uint32_t a0, a1, a2, a3, b0, b1, e0, e1, e2, e3, f0, f1;
            ldsm_x4(a_base + 32u * ks, a0, a1, a2, a3);
            ldsm_x2(b_base + b_step * ks, b0, b1);
            ldsm_x4(a_base + 32u * (ks + 1), e0, e1, e2, e3);
            ldsm_x2(b_base + b_step * (ks + 1), f0, f1);
            mma_16816(acc0, a0, a1, a2, a3, b0, b1);
            mma_16816(acc1, e0, e1, e2, e3, f0, f1);
          }
          if (ks < KS) {
            uint32_t a0, a1, a2, a3, b0, b1;
            ldsm_x4(a_base + 32u * ks, a0, a1, a2, a3);
            ldsm_x2(b_base + b_step * ks, b0, b1);
            mma_16816(acc0, a0, a1, a2, a3, b0, b1);
          }
          // thread (g, t4): rows g and g+8, columns 2*t4 (hi) and 2*t4+1 (lo) = token t4
          const int g = lane >> 2, t4 = lane & 3;
          const float s_g = (acc0[0] + acc1[0]) + (acc0[1] + acc1[1]);
          const float s_g8 = (acc0[2] + acc1[2]) + (acc0[3] + acc1[3]);
          const int r0 = 16 * it + g, r8 = r0 + 8;
          bool on0 = t4 < B && g < rows && (s_g + s.bp[r0]) > Ly.thr;
          bool on8 = t4 < B && g + 8 < rows && (s_g8 + s.bp[r8 < nrows ? r8 : r0]) > Ly.thr;
          on0 |= __shfl_xor_sync(0xffffffffu, on0, 1);
          on0 |= __shfl_xor_sync(0xffffffffu, on0, 2);
          on8 |= __shfl_xor_sync(0xffffffffu, on8, 1);
          on8 |= __shfl_xor_sync(0xffffffffu, on8, 2);
          if (t4 == 0) {
            if (g < rows) s.act[r0] = on0 ? 1 : 0;
            if (g + 8 < rows) s.act[r8] = on8 ? 1 : 0;
          }
        }
        release_item();
      }
      witem += ntile;
    } else {
      const int nu = r / 8;  // 8-element units per row (r % 8 == 0)
      // single token and rank <= 1024: this lane's slice of u stays in registers
      float ureg[4][8];
      const bool u_in_regs = (B == 1) && nu <= 128;
      if (u_in_regs) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int m = lane + 32 * i;
          float4 lo = make_float4(0.f, 0.f, 0.f, 0.f), hi = lo;
          if (m < nu) {
            lo = reinterpret_cast<const float4*>(s.u)[m];
            hi = reinterpret_cast<const float4*>(s.u)[nu + m];
          }
          ureg[i][0] = lo.x; ureg[i][1] = lo.y; ureg[i][2] = lo.z; ureg[i][3] = lo.w;
          ureg[i][4] = hi.x; ureg[i][5] = hi.y; ureg[i][6] = hi.z; ureg[i][7] = hi.w;
        }
      }
      for (int cc = c0; cc < c1; cc += NW) {
        const int rows = min(NW, c1 - cc);
        uint32_t off;
        to |= !wait_item(off);
        if (warp < rows) {
          const uint8_t* row = s.ring + off + (size_t)warp * r * ep;
          float acc[B];
#pragma unroll
          for (int b = 0; b < B; ++b) acc[b] = 0.f;
          if (u_in_regs) {
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int m = lane + 32 * i;
              if (m < nu) {
                float w[8];
                if constexpr (PT == kF16) {
                  const uint4 q = *reinterpret_cast<const uint4*>(row + 16 * m);
                  float2 f;
                  f = h2f2(q.x); w[0] = f.x; w[1] = f.y;
                  f = h2f2(q.y); w[2] = f.x; w[3] = f.y;
                  f = h2f2(q.z); w[4] = f.x; w[5] = f.y;
                  f = h2f2(q.w); w[6] = f.x; w[7] = f.y;
                } else {
                  const float4 a = *reinterpret_cast<const float4*>(row + 32 * m);
                  const float4 b2 = *reinterpret_cast<const float4*>(row + 32 * m + 16);
                  w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
                  w[4] = b2.x; w[5] = b2.y; w[6] = b2.z; w[7] = b2.w;
                }
                a0 = fmaf(w[0], ureg[i][0], a0); a1 = fmaf(w[1], ureg[i][1], a1);
                a0 = fmaf(w[2], ureg[i][2], a0); a1 = fmaf(w[3], ureg[i][3], a1);
                a0 = fmaf(w[4], ureg[i][4], a0); a1 = fmaf(w[5], ureg[i][5], a1);
                a0 = fmaf(w[6], ureg[i][6], a0); a1 = fmaf(w[7], ureg[i][7], a1);
              }
            }
            acc[0] = a0 + a1;
          } else
#pragma unroll 2
          for (int m = lane; m < nu; m += 32) {
            float w[8];
            if constexpr (PT == kF16) {
              const uint4 q = *reinterpret_cast<const uint4*>(row + 16 * m);
              float2 f;
              f = h2f2(q.x); w[0] = f.x; w[1] = f.y;
              f = h2f2(q.y); w[2] = f.x; w[3] = f.y;
              f = h2f2(q.z); w[4] = f.x; w[5] = f.y;
              f = h2f2(q.w); w[6] = f.x; w[7] = f.y;
            } else {
              const float4 a = *reinterpret_cast<const float4*>(row + 32 * m);
              const float4 b2 = *reinterpret_cast<const float4*>(row + 32 * m + 16);
              w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
              w[4] = b2.x; w[5] = b2.y; w[6] = b2.z; w[7] = b2.w;
            }
#pragma unroll
            for (int b = 0; b < B; ++b) {
              const float4* ub = reinterpret_cast<const float4*>(s.u + (size_t)b * r);
              const float4 lo = ub[m], hi = ub[nu + m];
              float a = acc[b];
              a = fmaf(w[0], lo.x, a); a = fmaf(w[1], lo.y, a); a = fmaf(w[2], lo.z, a); a = fmaf(w[3], lo.w, a);
              a = fmaf(w[4], hi.x, a); a = fmaf(w[5], hi.y, a); a = fmaf(w[6], hi.z, a); a = fmaf(w[7], hi.w, a);
              acc[b] = a;
            }
          }
          bool on = false;
          const float bias = s.bp[cc - c0 + warp];
#pragma unroll
          for (int b = 0; b < B; ++b) on |= (warp_sum(acc[b]) + bias) > Ly.thr;
          if (lane == 0) s.act[cc - c0 + warp] = on ? 1 : 0;
        }
        release_item();
      }
    }
    if (named_sync_or(1, T, to)) return;
    // local ascending list of this CTA's active cold rows (consumer warp 0)
    if (warp == 0) {
      int cnt = 0;
      for (int x0 = 0; x0 < c1 - c0; x0 += 32) {
        const int x = x0 + lane;
        const bool on = x < c1 - c0 && s.act[x];
        const unsigned m = __ballot_sync(0xffffffffu, on);
        if (on) p.seg[(int64_t)c * p.seg_cap + cnt + __popc(m & ((1u << lane) - 1u))] = H + c0 + x;
        cnt += __popc(m);
      }
      if (lane == 0) p.seg_cnt[c] = cnt;
      __syncwarp();
      if (lane == 0) grid_arrive(ctrl);
    }

    // ---- sparse FFN: hot share, then cold share, two neurons in flight ----
#pragma unroll
    for (int b = 0; b < B; ++b)
#pragma unroll
      for (int e = 0; e < EPT; ++e) y[b][e] = 0.f;
    const int wrp = wrow_bytes(WT, d) + 16;  // byte stride of a neuron item's rows
    const int nh = j1 - j0;
    int n = nh;
    bool have_list = false;
    uint32_t itoff0 = 0u, itoff1 = 0u;
    float* nred = s.red + 2 * (kMaxConsumers / 32) * (4 * B);  // neuron scratch: [2][NW][2B]
    // dots of neuron k -> per-warp partial sums in nred[k & 1]
    auto prepare = [&](int k) {
      uint32_t off;
      to |= !wait_item(off);
      if (k & 1) itoff1 = off;
      else itoff0 = off;
      const uint8_t* it = s.ring + off;
      float acc[2 * B];
      float wu[EPT];
      w_vals<WT, EPT>(it + (gated ? wrp : 0), d, t, T, wu);
#pragma unroll
      for (int b = 0; b < B; ++b) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < EPT; ++e) a = fmaf(wu[e], h[b][e], a);
        acc[B + b] = a;
      }
      if (gated) {
        float wg[EPT];
        w_vals<WT, EPT>(it, d, t, T, wg);
#pragma unroll
        for (int b = 0; b < B; ++b) {
          float a = 0.f;
#pragma unroll
          for (int e = 0; e < EPT; ++e) a = fmaf(wg[e], h[b][e], a);
          acc[b] = a;
        }
      } else {
#pragma unroll
        for (int b = 0; b < B; ++b) acc[b] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 2 * B; ++i) acc[i] = warp_sum(acc[i]);
      float* red = nred + (k & 1) * (kMaxConsumers / 32) * (2 * B);
      if (lane == 0) {
#pragma unroll
        for (int i = 0; i < 2 * B; ++i) red[warp * 2 * B + i] = acc[i];
      }
    };
    // activation and down-row accumulation of neuron k (after its barrier)
    auto finish = [&](int k) {
      const float* red = nred + (k & 1) * (kMaxConsumers / 32) * (2 * B);
      float tot[2 * B];
#pragma unroll
      for (int i = 0; i < 2 * B; ++i) {
        float v = lane < NW ? red[lane * 2 * B + i] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        tot[i] = v;
      }
      const float bias = k < nh ? s.b1hot[k] : s.cb1[k - nh];
      float a[B];
#pragma unroll
      for (int b = 0; b < B; ++b)
        a[b] = gated ? act_eval(kReglu, tot[b] + bias, tot[B + b]) : act_eval(p.act, tot[B + b] + bias, 0.f);
      float wd[EPT];
      w_vals<WT, EPT>(s.ring + ((k & 1) ? itoff1 : itoff0) + (gated ? 2 : 1) * wrp, d, t, T, wd);
      release_item();
#pragma unroll
      for (int b = 0; b < B; ++b)
#pragma unroll
        for (int e = 0; e < EPT; ++e) y[b][e] = fmaf(a[b], wd[e], y[b][e]);
    };
    // the cold list (and its biases) from the producer
    auto take_list = [&]() -> bool {
      const bool okw = mbar_wait(s.list_bar, l & 1, ctrl);
      if (named_sync_or(1, T, !okw)) return false;
      const int ncold = s.misc[0];
      for (int x = t; x < ncold; x += T) s.cb1[x] = Ly.b1 ? __ldg(Ly.b1 + s.cidx[x]) : 0.f;
      n = nh + ncold;
      have_list = true;
      return true;
    };
    if constexpr (WT == kF16 && PT == kF16) {
      // Tensor cores for the gate/up dots of p.ng neurons at a time: their
      // gate and up rows form one 16-row A tile (unused rows repeat neuron 0),
      // the fp16 token rows the B tile; warps split d and their partial dots
      // meet in shared memory, one thread per (neuron, token) applies the
      // activation, then every thread adds the group's down rows into its
      // columns of the partial output.
      const int rpn = gated ? 2 : 1;  // tile rows per neuron
      const int bn = lane & 7;
      const uint32_t b_base =
          bn < B ? smem_u32(s.hb + bn * HS) + (uint32_t)(((lane >> 3) & 1) * 16) : smem_u32(s.zero);
      const uint32_t b_step = bn < B ? 32u : 0u;
      const int KS = d / 16, ks0 = warp * KS / NW, ks1 = (warp + 1) * KS / NW;
      float* gact = nred;  // [ng][B] activations of the group
      int k = 0;
      for (;;) {
        if (k == nh && !have_list) {
          if (!take_list()) return;
          named_sync(1, T);  // cb1 visible
        }
        const int lim = have_list ? n : nh;
        if (k >= lim) break;
        const int ng = min(p.ng, lim - k);
        for (int i = 0; i < ng; ++i) to |= !mbar_wait(&s.full[(witem + i) % kNQ], ((witem + i) / kNQ) & 1u, ctrl);
        if (!to) {
          const int tr = lane & 15;
          const int jj = tr / rpn < ng ? tr / rpn : 0;
          const int which = gated ? (tr & 1) : 0;  // item row: gate then up (ReGLU), up (otherwise)
          const uint32_t a_base = smem_u32(s.ring + s.item_off[(witem + jj) % kNQ]) + (uint32_t)(which * wrp) +
                                  (uint32_t)((lane >> 4) * 16);
          float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
          int ks = ks0;
          for (; ks + 1 < ks1; ks += 2) {
            uint32_t a0, a1, a2, a3, b0, b1, e0, e1, e2, e3, f0, f1;
            ldsm_x4(a_base + 32u * ks, a0, a1, a2, a3);
            ldsm_x2(b_base + b_step * ks, b0, b1);
            ldsm_x4(a_base + 32u * (ks + 1), e0, e1, e2, e3);
            ldsm_x2(b_base + b_step * (ks + 1), f0, f1);
            mma_16816(acc0, a0, a1, a2, a3, b0, b1);
            mma_16816(acc1, e0, e1, e2, e3, f0, f1);
          }
          if (ks < ks1) {
            uint32_t a0, a1, a2, a3, b0, b1;
            ldsm_x4(a_base + 32u * ks, a0, a1, a2, a3);
            ldsm_x2(b_base + b_step * ks, b0, b1);
            mma_16816(acc0, a0, a1, a2, a3, b0, b1);
          }
          // thread (g = lane/4, lane%4 == 0) holds tile rows g and g+8, tokens 0 and 1
          if ((lane & 3) == 0) {
            const int g = lane >> 2;
            float* rp = s.redp + warp * 32;
            rp[g * 2 + 0] = acc0[0] + acc1[0];
            rp[g * 2 + 1] = acc0[1] + acc1[1];
            rp[(g + 8) * 2 + 0] = acc0[2] + acc1[2];
            rp[(g + 8) * 2 + 1] = acc0[3] + acc1[3];
          }
        }
        if (named_sync_or(1, T, to)) return;
        if (t < ng * B) {
          const int jj = t / B, b = t % B;
          float gd = 0.f, vd = 0.f;
          for (int w = 0; w < NW; ++w) {
            gd += s.redp[w * 32 + (jj * rpn) * 2 + b];
            vd += s.redp[w * 32 + (jj * rpn + rpn - 1) * 2 + b];
          }
          const int kk = k + jj;
          const float bias = kk < nh ? s.b1hot[kk] : s.cb1[kk - nh];
          gact[jj * B + b] = gated ? act_eval(kReglu, gd + bias, vd) : act_eval(p.act, vd + bias, 0.f);
        }
        named_sync(1, T);
        for (int jj = 0; jj < ng; ++jj) {
          float wd[EPT];
          w_vals<WT, EPT>(s.ring + s.item_off[(witem + jj) % kNQ] + rpn * wrp, d, t, T, wd);
#pragma unroll
          for (int b = 0; b < B; ++b) {
            const float a = gact[jj * B + b];
#pragma unroll
            for (int e = 0; e < EPT; ++e) y[b][e] = fmaf(a, wd[e], y[b][e]);
          }
        }
        witem += ng;
        for (int i = 0; i < ng; ++i) release_item();
        k += ng;
      }
    } else {
      if (nh == 0) {
        if (!take_list()) return;
        named_sync(1, T);  // cb1 visible
      }
      if (n > 0) prepare(0);
      for (int k = 0; k < n; ++k) {
        if (named_sync_or(1, T, to)) return;  // neuron k's partial sums are complete
        if (k + 1 == nh && !have_list) {
          if (!take_list()) return;  // cb1 becomes visible at the next neuron's barrier
        }
        if (k + 1 < n) prepare(k + 1);
        finish(k);
      }
      if (!have_list) {  // (nh > 0 and the loop ended before the list: cannot happen, kept for safety)
        if (!take_list()) return;
      }
    }

    // ---- split-K: add the partial into one of K fp32 accumulator copies ----
    {
      float* acc = p.yacc + ((size_t)(l & 1) * K + (c % K)) * B * d;
      using O = Own<WT, EPT>;
#pragma unroll
      for (int b = 0; b < B; ++b)
#pragma unroll
        for (int k = 0; k < O::NRUN; ++k) {
          const int col = O::col(t, T, k);
#pragma unroll
          for (int e = 0; e < O::RUN; e += 4)
            atomicAdd(reinterpret_cast<float4*>(acc + (size_t)b * d + col + e),
                      make_float4(y[b][k * O::RUN + e], y[b][k * O::RUN + e + 1], y[b][k * O::RUN + e + 2],
                                  y[b][k * O::RUN + e + 3]));
        }
    }
    named_sync(1, T);
    if (t == 0) grid_arrive(ctrl);
    {
      bool okw = true;
      if (t == 0) okw = grid_wait(ctrl, base, 3 * l + 2, G);
      if (named_sync_or(1, T, !okw)) return;
    }

    // ---- glue: h <- RMSNorm(h + y + b2), rounded to the token type ----
    {
      const float* acc = p.yacc + (size_t)(l & 1) * K * B * d;
      using O = Own<WT, EPT>;
      float ss[B];
#pragma unroll
      for (int b = 0; b < B; ++b) {
        float yv[EPT];
#pragma unroll
        for (int k = 0; k < O::NRUN; ++k) {
          const int col = O::col(t, T, k);
#pragma unroll
          for (int e = 0; e < O::RUN; e += 4) {
            float4 bb = make_float4(0.f, 0.f, 0.f, 0.f);
            if (Ly.b2) bb = __ldg(reinterpret_cast<const float4*>(Ly.b2 + col + e));
            float4 v[K];
#pragma unroll
            for (int q = 0; q < K; ++q)
              v[q] = __ldcg(reinterpret_cast<const float4*>(acc + ((size_t)q * B + b) * d + col + e));
#pragma unroll
            for (int q = 0; q < K; ++q) {
              bb.x += v[q].x; bb.y += v[q].y; bb.z += v[q].z; bb.w += v[q].w;
            }
            yv[k * O::RUN + e] = bb.x;
            yv[k * O::RUN + e + 1] = bb.y;
            yv[k * O::RUN + e + 2] = bb.z;
            yv[k * O::RUN + e + 3] = bb.w;
          }
        }
        if (c == 0 && p.y_out) store_vals<WT, EPT, kF32>(reinterpret_cast<uint8_t*>(p.y_out + ((size_t)l * B + b) * d), t, T, yv);
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < EPT; ++e) {
          const float x = h[b][e] + yv[e];
          h[b][e] = x;
          a = fmaf(x, x, a);
        }
        ss[b] = a;
      }
      cta_reduce<B, 4 * B>(ss, s.red, par, warp, lane, NW, T, false);
#pragma unroll
      for (int b = 0; b < B; ++b) {
        const float inv = rsqrtf(ss[b] / (float)d + p.eps);
#pragma unroll
        for (int e = 0; e < EPT; ++e) h[b][e] = round_to(PT, h[b][e] * inv);
      }
      if constexpr (PT == kF16) {
#pragma unroll
        for (int b = 0; b < B; ++b) store_vals<WT, EPT, kF16>(s.hb + b * HS, t, T, h[b]);
      }
      if (c == 0) {
        uint8_t* dst = nullptr;
        if (l + 1 < p.L) {
          if (p.h_trace) dst = reinterpret_cast<uint8_t*>(p.h_trace) + (size_t)(l + 1) * B * d * ep;
        } else {
          dst = reinterpret_cast<uint8_t*>(p.h_out);
        }
        if (dst) {
#pragma unroll
          for (int b = 0; b < B; ++b) store_vals<WT, EPT, PT>(dst + (size_t)b * d * ep, t, T, h[b]);
        }
      }
    }
  }
  // every CTA has passed the last barrier: leave the count base for the next launch
  if (c == 0 && t == 0) atomicExch(&ctrl->bar_base, base + (unsigned)(3 * p.L * G));
}

template <int WT, int PT, int B, int EPT>
cudaError_t launch_t(const StackParams& p, int G, size_t smem, cudaStream_t st) {
  auto fn = k_stack<WT, PT, B, EPT>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(p.T + 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fn, p);
}

}  // namespace

int stack_ept(int d) { return (d % 256 == 0 && d / 8 <= kMaxConsumers) ? 8 : 16; }

bool stack_supported(int wtype, int ptype, int d, int ffn, int n_hot, int rank, int B, int L) {
  if (B < 1 || B > 2) return false;
  if (L < 1 || L > kMaxLayers) return false;
  const bool combo = (wtype == kF16 && ptype == kF16) || (wtype == kQ4_0 && ptype == kF16) ||
                     (wtype == kF32 && ptype == kF32);
  if (!combo) return false;
  const int ept = stack_ept(d);
  if (d % (32 * ept) != 0 || d / ept > kMaxConsumers) return false;
  if (wtype == kQ4_0 && d % 256 != 0) return false;
  if (rank % 8 != 0 || rank > kMaxRank) return false;
  (void)ffn;
  (void)n_hot;
  return true;
}

size_t stack_smem_layout(StackParams& p, int B, int G) {
  const int C = p.ffn - p.n_hot;
  const int share_cap = (C + G - 1) / G + 1;
  const int hot_cap = (p.n_hot + G - 1) / G + 1;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 127) & ~(size_t)127;
    return (int)o;
  };
  // everything but the ring first (at the end of shared memory), then the ring
  size_t fixed = 0;
  {
    size_t o = 0;
    auto t2 = [&](size_t bytes) { o += (bytes + 127) & ~(size_t)127; };
    t2(sizeof(uint64_t) * (2 * kNQ + 1));
    t2(sizeof(uint32_t) * 3 * kNQ);
    t2(sizeof(float) * (size_t)B * p.rank);
    t2(sizeof(float) * share_cap);
    t2(sizeof(float) * hot_cap);
    t2(sizeof(int) * share_cap);
    t2(sizeof(float) * share_cap);
    t2(share_cap);
    t2(sizeof(float) * 2 * (kMaxConsumers / 32) * 6 * B);
    t2(sizeof(int) * (G + 1));
    t2(sizeof(int) * 4);
    t2((size_t)B * (2 * p.d + 16));
    t2((size_t)2 * B * (2 * p.rank + 16));
    t2(16);
    t2(sizeof(float) * (kMaxConsumers / 32) * 32);
    fixed = o;
  }
  const size_t total = kSmemBytes;
  if (fixed + 32768 > total) return 0;
  const size_t ring = (total - fixed) & ~(size_t)127;
  p.ring_bytes = (int)ring;
  off = ring;
  p.off_bars = take(sizeof(uint64_t) * (2 * kNQ + 1));
  p.off_itemoff = take(sizeof(uint32_t) * 3 * kNQ);
  p.off_u = take(sizeof(float) * (size_t)B * p.rank);
  p.off_bp = take(sizeof(float) * share_cap);
  p.off_b1hot = take(sizeof(float) * hot_cap);
  p.off_cidx = take(sizeof(int) * share_cap);
  p.off_cb1 = take(sizeof(float) * share_cap);
  p.off_act = take(share_cap);
  p.off_red = take(sizeof(float) * 2 * (kMaxConsumers / 32) * 6 * B);
  p.off_prefix = take(sizeof(int) * (G + 1));
  p.off_misc = take(sizeof(int) * 4);
  p.off_hb = take((size_t)B * (2 * p.d + 16));
  p.off_ub = take((size_t)2 * B * (2 * p.rank + 16));
  p.off_zero = take(16);
  p.off_redp = take(sizeof(float) * (kMaxConsumers / 32) * 32);
  return off;
}

cudaError_t launch_stack(int wtype, int ptype, int B, const StackParams& p, int G, size_t smem, cudaStream_t st) {
  const int ept = p.d / p.T;
#define PI_STACK_CASE(W_, P_, B_, E_) \
  if (wtype == W_ && ptype == P_ && B == B_ && ept == E_) return launch_t<W_, P_, B_, E_>(p, G, smem, st);
  PI_STACK_CASE(kF16, kF16, 1, 8)
  PI_STACK_CASE(kF16, kF16, 2, 8)
  PI_STACK_CASE(kF16, kF16, 1, 16)
  PI_STACK_CASE(kF16, kF16, 2, 16)
  PI_STACK_CASE(kQ4_0, kF16, 1, 8)
  PI_STACK_CASE(kQ4_0, kF16, 2, 8)
  PI_STACK_CASE(kQ4_0, kF16, 1, 16)
  PI_STACK_CASE(kQ4_0, kF16, 2, 16)
  PI_STACK_CASE(kF32, kF32, 1, 8)
  PI_STACK_CASE(kF32, kF32, 2, 8)
  PI_STACK_CASE(kF32, kF32, 1, 16)
  PI_STACK_CASE(kF32, kF32, 2, 16)
#undef PI_STACK_CASE
  return cudaErrorInvalidValue;
}

}  // namespace pi
