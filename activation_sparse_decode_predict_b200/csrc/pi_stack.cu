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
//     consumption order per layer: its P1 rows, a static share of the hot
//     neurons, its block of P2 rows, then a stream of neurons: the cold rows
//     its own CTA predicted active (an excess over its running mean is handed
//     to the other CTAs) and chunks of the remaining hot neurons claimed from
//     a per-layer atomic counter (the claims balance the per-CTA cold
//     counts).  A neuron item is its gate/up/down rows plus the 16-byte block
//     of b1 that holds its bias.
//   * consumer warps own fixed columns of d: the token block and the fp32
//     partial output stay in registers for the whole layer.  The neuron dots
//     (and the P1 dots of a single token) run on CUDA cores, P2 (and the P1
//     of a token block of 2) on the tensor cores with mma.sync.
//   * per layer: P1 rows -> u (global) -> barrier U (static hot neurons fill
//     the wait) -> P2 scores of the CTA's cold rows -> local ascending list ->
//     neuron stream -> partial y added into an fp32 accumulator with vector
//     atomics -> barrier Y -> residual + RMSNorm glue computed redundantly by
//     every CTA -> next layer.  Two grid barriers per layer.
//   * the ascending list pi_predict would write is each CTA's local list in
//     CTA order; every CTA parks its list in place and the lists are
//     compacted once, after the last layer.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "pi_common.cuh"
#include "pi_mma.cuh"
#include "pi_stack.cuh"
#include "pi_sync.cuh"

// PI_TRACE builds record %globaltimer stamps at the phase boundaries of every
// layer and CTA into p.trace (a profiling aid; the default build has none).
#ifdef PI_TRACE
#define PI_STAMP(l, e) \
  do { if (p.trace) p.trace[((size_t)(l) * gridDim.x + blockIdx.x) * kTraceEvents + (e)] = global_ns(); } while (0)
#define PI_STAMP_VAL(l, e, v) \
  do { if (p.trace) p.trace[((size_t)(l) * gridDim.x + blockIdx.x) * kTraceEvents + (e)] = (uint64_t)(v); } while (0)
#else
#define PI_STAMP(l, e) do { } while (0)
#define PI_STAMP_VAL(l, e, v) do { } while (0)
#endif

namespace pi {

namespace {

// Warp sums of V values per lane with V - 1 + 5 - log2(V) shuffles: every
// exchange step halves the values a lane keeps.  The sum of value i ends in
// lanes whose bits 4..(5 - log2 V) spell i, so lane i * (32 / V) holds it.
template <int V>
__device__ __forceinline__ float warp_sums(const float (&v)[V], int lane) {
  static_assert(V == 2 || V == 4, "2 or 4 values");
  const bool h16 = (lane & 16) != 0;
  if constexpr (V == 2) {
    float k = h16 ? v[1] : v[0];
    k += __shfl_xor_sync(0xffffffffu, h16 ? v[0] : v[1], 16);
#pragma unroll
    for (int o = 8; o; o >>= 1) k += __shfl_xor_sync(0xffffffffu, k, o);
    return k;
  } else {
    float k0 = h16 ? v[2] : v[0], k1 = h16 ? v[3] : v[1];
    k0 += __shfl_xor_sync(0xffffffffu, h16 ? v[0] : v[2], 16);
    k1 += __shfl_xor_sync(0xffffffffu, h16 ? v[1] : v[3], 16);
    const bool h8 = (lane & 8) != 0;
    float k = h8 ? k1 : k0;
    k += __shfl_xor_sync(0xffffffffu, h8 ? k0 : k1, 8);
#pragma unroll
    for (int o = 4; o; o >>= 1) k += __shfl_xor_sync(0xffffffffu, k, o);
    return k;
  }
}

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

// This thread's Q4_0 codes as f = 1 + q/16 (q placed in the top mantissa
// bits of 1.0f: exact, no integer-to-float conversion), so q - 8 = 16 f - 24;
// sc is the block's scale.  A dot over the thread's columns is then
// sc * (16 * sum(f h) - 24 * sum(h)).
template <int EPT>
__device__ __forceinline__ void q4_codes(const uint8_t* row, int d, int t, float (&f)[EPT], float& sc) {
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
  sc = half_bits_to_float(*reinterpret_cast<const uint16_t*>(row + d / 2 + 2 * (t / PER_BLK)));
#pragma unroll
  for (int w = 0; w < NB / 4; ++w)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t b = q[w] >> (8 * k);
      f[w * 4 + k] = __uint_as_float(0x3f800000u | ((b & 0xfu) << 19));
      f[NB + w * 4 + k] = __uint_as_float(0x3f800000u | ((b & 0xf0u) << 15));
    }
}

// The thread's EPT values of an fp16 or fp32 weight row (Q4_0 rows are read
// with q4_codes).
template <int WT, int EPT>
__device__ __forceinline__ void w_vals(const uint8_t* row, int t, int T, float (&v)[EPT]) {
  static_assert(WT != kQ4_0, "Q4_0 rows are read with q4_codes");
  row_vals<WT, EPT, WT>(row, t, T, v);
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

__device__ __forceinline__ int wrow_bytes(int WT_, int d) {
  return WT_ == kQ4_0 ? d / 2 + d / 16 : d * (WT_ == kF16 ? 2 : 4);
}

struct Smem {
  uint8_t* ring;
  uint64_t* full;
  uint64_t* empty;
  uint64_t* list_bar;
  uint64_t* u_bar;   // consumers -> barrier warp: this layer's u rows are written
  uint64_t* u_ready; // barrier warp -> consumers: barrier U passed, every CTA's u is staged
  uint32_t* item_off;
  uint32_t* istart;  // producer-private: start of the items in flight
  int* item_j;       // neuron row of a neuron item; -1 for an end marker
  int* item_gs;      // on the first item of a group: the group's size (0: end marker)
  float* u;          // [B][r] split layout (see load_u)
  float* bp;
  int* cidx;         // this CTA's predicted-active cold rows (neuron ids), ascending
  uint8_t* act;
  float* sc;         // partial P2 scores [k-part][rows][B]
  float* red;        // [2][NW][2B]
  float* gred;       // [kMaxGroup][NW][2B] per-warp gate/up dots (CUDA-core groups)
  int* misc;         // [0] local cold count, [1] barrier base, [2] next group size, [3] scratch
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
  s.u_bar = s.list_bar + 1;
  s.u_ready = s.list_bar + 2;
  s.item_off = reinterpret_cast<uint32_t*>(base + p.off_itemoff);
  s.istart = s.item_off + kNQ;
  s.item_j = reinterpret_cast<int*>(s.item_off + 2 * kNQ);
  s.item_gs = reinterpret_cast<int*>(s.item_off + 3 * kNQ);
  s.u = reinterpret_cast<float*>(base + p.off_u);
  s.bp = reinterpret_cast<float*>(base + p.off_bp);
  s.cidx = reinterpret_cast<int*>(base + p.off_cidx);
  s.act = base + p.off_act;
  s.sc = reinterpret_cast<float*>(base + p.off_sc);
  s.red = reinterpret_cast<float*>(base + p.off_red);
  s.gred = reinterpret_cast<float*>(base + p.off_gred);
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

  // One neuron: its gate (ReGLU only), up and down rows, then (with a b1)
  // the 16-byte block of b1 that holds its bias.  Row m of the item starts
  // m * (wrb + 16) bytes past a 128-byte aligned base that is shifted by
  // 32 * (neuron sequence number mod 4) bytes, so that the gate and up rows
  // of four consecutive neurons fall on eight different shared-memory bank
  // groups (conflict-free ldmatrix).  Q4_0 rows hold qs then sc.  gs > 0
  // marks the first item of a group of gs neurons.
  uint32_t nseq = 0;
  __device__ bool issue_neuron(const StackLayer& Ly, int j, int wt, int gated, int gs) {
    const int d = p.d;
    const uint32_t wrb = wt == kQ4_0 ? (uint32_t)(d / 2 + d / 16) : (uint32_t)(d * (wt == kF16 ? 2 : 4));
    const uint32_t wrp = wrb + 16;
    const int nrow = gated ? 3 : 2;
    const uint32_t skew = 32u * (nseq & 3u);
    ++nseq;
    const uint32_t total = nrow * wrp + 16 + 128 + skew;
    uint32_t pos;
    if (!alloc(total, pos)) return false;
    const uint32_t start = ((pos + 127u) & ~127u) + skew;
    const uint32_t q = item % kNQ;
    s.item_off[q] = start;
    s.istart[q] = pos;
    s.item_j[q] = j;
    s.item_gs[q] = gs;
    mbar_arrive_expect_tx(&s.full[q], nrow * wrb + (Ly.b1 ? 16u : 0u));
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
    if (Ly.b1) bulk_g2s(s.ring + start + nrow * wrp, Ly.b1 + (j & ~3), 16u, &s.full[q]);
    head = pos + total;
    ++item;
    return true;
  }

  // One group of gs neurons: rows j0 .. j0+gs-1, or list[0 .. gs)
  __device__ bool issue_group(const StackLayer& Ly, int j0, const int* list, int gs, int wt, int gated) {
    bool ok = true;
    for (int i = 0; i < gs && ok; ++i) ok = issue_neuron(Ly, list ? list[i] : j0 + i, wt, gated, i == 0 ? gs : 0);
    return ok;
  }

  // neurons j0 .. j0+n-1 in groups of at most ng
  __device__ bool issue_range(const StackLayer& Ly, int j0, int n, int wt, int gated) {
    bool ok = true;
    for (int i = 0; i < n && ok; i += p.ng) ok = issue_group(Ly, j0 + i, nullptr, min(p.ng, n - i), wt, gated);
    return ok;
  }

  // Ticket tk on layer l's handed-over cold rows: the row, or -1 once every CTA
  // has decided and the ticket is past the last slot (bounded waits).
  __device__ int take_donated(int l, unsigned tk, int C, int G) {
    const uint64_t t0 = global_ns();
    for (uint32_t it = 0;; ++it) {
      const unsigned pushed = ld_relaxed_u32(&ctrl->don_push[l]);
      if (tk < pushed) {
        const int v = ld_volatile_s32(p.don + (size_t)l * C + tk);
        if (v != 0) {
          // a handed-over row is a cold row of this layer; anything else is
          // reported and dropped (the workspace was not initialised)
          if (v - 1 < p.n_hot || v - 1 >= p.ffn) {
            set_status(&ctrl->status, kStIndex);
            return -1;
          }
          return v - 1;
        }
      } else if (ld_acquire_u32(&ctrl->don_done[l]) == (unsigned)G) {
        // every reservation happened before its CTA's release of don_done
        if (tk >= ld_relaxed_u32(&ctrl->don_push[l])) return -1;
        continue;
      }
      if ((it & 31u) == 0) {
        if (ld_volatile_s32(&ctrl->abort)) return -2;
        if (global_ns() - t0 > kTimeoutNs) {
          raise_abort(ctrl);
          return -2;
        }
      }
    }
  }

  // End of a neuron stream: an item without bytes (group size 0).
  __device__ bool issue_marker() {
    uint32_t pos;
    if (!alloc(0, pos)) return false;
    const uint32_t q = item % kNQ;
    s.item_off[q] = pos;
    s.istart[q] = pos;
    s.item_j[q] = -1;
    s.item_gs[q] = 0;
    mbar_arrive(&s.full[q]);
    head = pos;
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
// 96 registers: with 17 or 18 warps per CTA an SM sub-partition holds 5 warps
__global__ void __maxnreg__(96) k_stack(const __grid_constant__ StackParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem s = carve(smem_raw, p);
  Ctrl* ctrl = p.ctrl;
  const int G = gridDim.x, c = blockIdx.x;
  const int T = p.T, NW = T / 32;
  const int d = p.d, H = p.n_hot, C = p.ffn - p.n_hot;
  const int gated = p.act == kReglu;
  // the token block is fp32 with fp32 predictors, fp16 with fp16 or Q4_0 ones
  constexpr int HT = PT == kF32 ? kF32 : kF16;
  const int ep = HT == kF16 ? 2 : 4;  // bytes per token element (and per fp16/fp32 predictor element)
  constexpr int K = kYCopies;
  // the fp16 token rows in shared memory feed only the tensor-core P1 (token
  // blocks of 2) and tensor-core neuron groups; otherwise they take no space
  constexpr bool kTokRows = stack_token_rows(PT, B);

  if (threadIdx.x == 0) {
    for (int q = 0; q < kNQ; ++q) {
      mbar_init(&s.full[q], 1);
      mbar_init(&s.empty[q], NW);
      s.item_off[q] = 0u;  // in-ring offsets even before the first item of a slot
      s.istart[q] = 0u;
    }
    mbar_init(s.list_bar, 1);
    mbar_init(s.u_bar, 1);
    mbar_init(s.u_ready, 1);
    mbar_fence_init();
    s.misc[1] = (int)ld_acquire_u32(&ctrl->bar_base);
  }
  __syncthreads();
  const unsigned base = (unsigned)s.misc[1];

  // shares that do not depend on the predictor (the P1 rows, a share of the
  // layer's rank, are taken per layer: each layer has its own rank)
  const int c0 = share_lo(C, c, G), c1 = share_lo(C, c + 1, G);

  // static hot share (consumed while barrier U completes); the rest of the
  // hot neurons, [HA, H), is claimed in chunks through p.pool[l]
  const int HA = p.hot_static;
  const int ha0 = share_lo(p.hot_a, c, G), ha1 = share_lo(p.hot_a, c + 1, G);  // before barrier U
  const int hb0 = p.hot_a + share_lo(HA - p.hot_a, c, G), hb1 = p.hot_a + share_lo(HA - p.hot_a, c + 1, G);

  if (threadIdx.x >= 32 + T) {
    // ======================= barrier warp =======================
    // Barrier U for the CTA: once the consumers have written their u rows it
    // arrives (the release waits for those writes to reach L2), waits for the
    // other CTAs and stages every CTA's u in shared memory, while the
    // consumers run the first static hot neurons.
    const int lane = threadIdx.x & 31;
    for (int l = 0; l < p.L; ++l) {
      const int r = p.layers[l].rank;
      const int US = 2 * r + 16;
      bool ok = true;
      if (lane == 0) {
        ok = mbar_wait(s.u_bar, l & 1, ctrl);
        PI_STAMP(l, 10);
        if (ok) grid_arrive(ctrl);
        if (ok) ok = grid_wait(ctrl, base, 2 * l, G);
        PI_STAMP(l, 11);
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) return;
      if constexpr (PT == kF16) {
        // row 2b = hi(u_b), row 2b+1 = lo(u_b) = u_b - hi: the tensor cores see ~22 bits of u
        // 16 loads per lane in flight at a time
        const int n2 = B * r / 2;
        for (int i0 = lane; i0 < n2; i0 += 32 * 16) {
          float2 v[16];
#pragma unroll
          for (int k = 0; k < 16; ++k)
            if (i0 + 32 * k < n2) v[k] = __ldcg(reinterpret_cast<const float2*>(p.u_g) + i0 + 32 * k);
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int i = i0 + 32 * k;
            if (i < n2) {
              const int b = (2 * i) / r, col = (2 * i) % r;
              const __half2 hi = __floats2half2_rn(v[k].x, v[k].y);
              const float2 hf = __half22float2(hi);
              const __half2 lo = __floats2half2_rn(v[k].x - hf.x, v[k].y - hf.y);
              *reinterpret_cast<__half2*>(s.ub + (2 * b) * US + 2 * col) = hi;
              *reinterpret_cast<__half2*>(s.ub + (2 * b + 1) * US + 2 * col) = lo;
            }
          }
        }
      } else if constexpr (PT == kQ4_0) {
        // Q4_0 P2 rows: lane m of a warp takes 32-element block m of a row, so
        // u is stored block-transposed, s.u[b][k][m] = u[b][32 m + k] with a
        // row stride of nblk + 1 (conflict-free writes and reads), and each
        // block's sum of u goes to s.usum[b][m] (see the Q4_0 row dot)
        const int nblk = r / 32, RS = 32 * (nblk + 1);
        float* usum = s.u + (size_t)B * (p.rank + 32);
        for (int i = lane; i < B * r; i += 32) {
          const int b = i / r, j = i % r;
          s.u[(size_t)b * RS + (j % 32) * (nblk + 1) + j / 32] = __ldcg(p.u_g + i);
        }
        __syncwarp();
        for (int i = lane; i < B * nblk; i += 32) {
          const int b = i / nblk, m = i % nblk;
          float a = 0.f;
          for (int kk = 0; kk < 32; ++kk) a += s.u[(size_t)b * RS + kk * (nblk + 1) + m];
          usum[i] = a;
        }
      } else {
        // split layout: unit m (8 values) stored as two float4 planes so that
        // lane-strided reads are conflict-free
        const int nu = r / 8;
        for (int i0 = lane; i0 < B * nu; i0 += 32 * 4) {
          float4 lo[4], hi[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int i = i0 + 32 * k;
            if (i < B * nu) {
              const float4* src = reinterpret_cast<const float4*>(p.u_g + (int64_t)(i / nu) * r + 8 * (i % nu));
              lo[k] = __ldcg(src);
              hi[k] = __ldcg(src + 1);
            }
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int i = i0 + 32 * k;
            if (i < B * nu) {
              const int b = i / nu, m = i % nu;
              float4* dst = reinterpret_cast<float4*>(s.u + (size_t)b * r);
              dst[m] = lo[k];
              dst[nu + m] = hi[k];
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(s.u_ready);
    }
    return;
  }

  if (threadIdx.x < 32) {
    // ======================= producer warp =======================
    const int lane = threadIdx.x;
    Producer pr(p, s);
    float cold_avg = 0.f;  // running mean of this CTA's predicted cold rows per layer
    bool ok = true;
    for (int l = 0; l < p.L && ok; ++l) {
      const StackLayer& Ly = p.layers[l];
      const int r = Ly.rank;
      const int k0 = share_lo(r, c, G), k1 = share_lo(r, c + 1, G);
      if (lane == 0) {
        // item order = consumption order
        if constexpr (PT == kF16) {
          // tensor-core predictor: skewed P1 rows, P2 in 16-row tiles with padded rows
          for (int k = k0; k < k1 && ok; ++k)
            ok = pr.issue_rows(reinterpret_cast<const uint8_t*>(Ly.P1) + (int64_t)k * d * 2, 0, 1, d * 2, d * 2,
                               16u * (uint32_t)((k - k0) & 7));
          if (ok) ok = pr.issue_range(Ly, ha0, ha1 - ha0, WT, gated);
          if (ok) ok = pr.issue_marker();
          for (int cc = c0; cc < c1 && ok; cc += 16)
            ok = pr.issue_rows(reinterpret_cast<const uint8_t*>(Ly.P2) + (int64_t)cc * r * 2, (int64_t)r * 2,
                               min(16, c1 - cc), r * 2, r * 2 + 16, 0);
        } else if constexpr (PT == kQ4_0) {
          // Q4_0 predictor rows: codes then scales, like a Q4_0 weight row
          for (int k = k0; k < k1 && ok; ++k) {
            const void* src[2] = {reinterpret_cast<const uint8_t*>(Ly.P1) + (int64_t)k * (d / 2),
                                  reinterpret_cast<const uint8_t*>(Ly.P1_sc) + (int64_t)k * (d / 16)};
            const uint32_t by[2] = {(uint32_t)(d / 2), (uint32_t)(d / 16)};
            ok = pr.issue(2, src, by);
          }
          if (ok) ok = pr.issue_range(Ly, ha0, ha1 - ha0, WT, gated);
          if (ok) ok = pr.issue_marker();
          // P2 items of NW rows: the rows' codes, then the rows' scales
          for (int cc = c0; cc < c1 && ok; cc += NW) {
            const int rows = min(NW, c1 - cc);
            const void* src[2] = {reinterpret_cast<const uint8_t*>(Ly.P2) + (int64_t)cc * (r / 2),
                                  reinterpret_cast<const uint8_t*>(Ly.P2_sc) + (int64_t)cc * (r / 16)};
            const uint32_t by[2] = {(uint32_t)(rows * (r / 2)), (uint32_t)(rows * (r / 16))};
            ok = pr.issue(2, src, by);
          }
        } else {
          for (int k = k0; k < k1 && ok; ++k) {
            const void* src = reinterpret_cast<const uint8_t*>(Ly.P1) + (int64_t)k * d * ep;
            const uint32_t by = d * ep;
            ok = pr.issue(1, &src, &by);
          }
          if (ok) ok = pr.issue_range(Ly, ha0, ha1 - ha0, WT, gated);
          if (ok) ok = pr.issue_marker();
          for (int cc = c0; cc < c1 && ok; cc += NW) {
            const int rows = min(NW, c1 - cc);
            const void* src = reinterpret_cast<const uint8_t*>(Ly.P2) + (int64_t)cc * r * ep;
            const uint32_t by = rows * r * ep;
            ok = pr.issue(1, &src, &by);
          }
        }
        // the neuron stream: one claimed hot chunk (covers the wait for the
        // local list), the predicted cold rows, more claimed chunks, the end marker
        // claim sizes shrink with what is left (guided self-scheduling): few
        // round trips early, fine balance at the end; one claim is in flight
        // while the previous one is issued
        const int PN = H - HA;
        int* pool = p.pool + l;
        // a claim is at least half a group, a whole one on wide rows (d >= 8192:
        // 40B-shaped +1.5 %, 70B-shaped +0.35 %; at 13B a whole group lost 2 %)
        const int cmin = d >= 8192 ? p.ng : max(1, p.ng / 2), cmax = 4 * p.ng;
        auto csize = [&](int seen) { return max(cmin, min(cmax, (PN - seen) / (2 * G))); };
        int nsz = csize(0);
        int nxt = PN > 0 ? atomicAdd(pool, nsz) : PN;
        if (hb1 > hb0) {
          if (ok) ok = pr.issue_range(Ly, hb0, hb1 - hb0, WT, gated);
        } else if (ok && nxt < PN) {
          const int cur = nxt, csz = nsz;
          nsz = csize(cur + csz);
          nxt = atomicAdd(pool, nsz);
          ok = pr.issue_range(Ly, HA + cur, min(csz, PN - cur), WT, gated);
        }
        if (ok) ok = mbar_wait(s.list_bar, l & 1, ctrl);
        const int nloc = s.misc[0];
        PI_STAMP(l, 12);
        PI_STAMP_VAL(l, 15, nloc);
        // A CTA with more predicted rows than its running mean (rounded up,
        // plus p.don_slack) hands the excess to the other CTAs (slots reserved with one atomic,
        // written as row + 1); every CTA takes handed-over rows by ticket once
        // its hot-neuron claims run out, until a ticket lands past the last
        // slot after every CTA has decided -- so no slot is left behind.
        int keep = nloc;
        if (kDonate && l > 0) keep = min(nloc, (int)ceilf(cold_avg) + p.don_slack);
        cold_avg = (l == 0) ? (float)nloc : 0.75f * cold_avg + 0.25f * (float)nloc;
        const int give = nloc - keep;
        if (give > 0) {
          const unsigned at = atomicAdd(&ctrl->don_push[l], (unsigned)give);
          for (int q = 0; q < give; ++q) st_volatile_s32(p.don + (size_t)l * C + at + q, s.cidx[keep + q] + 1);
        }
        red_release_add(&ctrl->don_done[l], 1u);
        for (int q = 0; q < keep && ok; q += p.ng) ok = pr.issue_group(Ly, 0, s.cidx + q, min(p.ng, keep - q), WT, gated);
        while (ok && nxt < PN) {
          const int cur = nxt, csz = nsz;
          // in the last round of chunks a CTA claims its next chunk only once
          // its own queue is short, so the last chunks go to the CTAs that are
          // about to run dry (kLazyTail)
          const bool tail = kLazyTail && PN - (cur + csz) < G * cmax;
          if (!tail) {
            nsz = csize(cur + csz);
            nxt = atomicAdd(pool, nsz);
          }
          ok = pr.issue_range(Ly, HA + cur, min(csz, PN - cur), WT, gated);
          if (tail) {
            while (ok && pr.item - pr.rel > (uint32_t)(kTailGroups * p.ng)) ok = pr.wait_consumed();
            nsz = csize(cur + csz);
            nxt = atomicAdd(pool, nsz);
          }
        }
        while (ok && C > 0) {
          if constexpr (kLazyTail)
            while (ok && pr.item - pr.rel > (uint32_t)(kTailGroups * p.ng)) ok = pr.wait_consumed();
          if (!ok) break;
          const int j = pr.take_donated(l, atomicAdd(&ctrl->don_take[l], 1u), C, G);
          if (j == -2) ok = false;
          if (j < 0) break;
          ok = pr.issue_group(Ly, j, nullptr, 1, WT, gated);
        }
        if (ok) ok = pr.issue_marker();
        PI_STAMP(l, 13);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
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
    row_vals<WT, EPT, HT>(reinterpret_cast<const uint8_t*>(p.h_in) + (int64_t)b * d * ep, t, T, h[b]);
  if (c == 0 && p.h_trace) {
#pragma unroll
    for (int b = 0; b < B; ++b) store_vals<WT, EPT, HT>(reinterpret_cast<uint8_t*>(p.h_trace) + (int64_t)b * d * ep, t, T, h[b]);
  }
  const int HS = 2 * d + 16;  // byte stride of the fp16 token rows in shared memory
  if constexpr (kTokRows) {
#pragma unroll
    for (int b = 0; b < B; ++b) store_vals<WT, EPT, kF16>(s.hb + b * HS, t, T, h[b]);
  }
  if constexpr (PT == kF16) {
    if (t < 4) reinterpret_cast<uint32_t*>(s.zero)[t] = 0u;
  }
  const int ybuf4 = K * B * d / 4;  // float4s per accumulator buffer (K copies)
  {
    const int z0 = share_lo(ybuf4, c, G), z1 = share_lo(ybuf4, c + 1, G);
    for (int i = z0 + t; i < z1; i += T) reinterpret_cast<float4*>(p.yacc)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }

  // the P2 biases of this CTA's cold rows: loaded one layer ahead into
  // registers, stored to shared memory after P1
  float bp_v[kShareRegs];
  auto load_shares = [&](const StackLayer& Lz) {
#pragma unroll
    for (int i = 0; i < kShareRegs; ++i) {
      const int x = t + i * T;
      bp_v[i] = (Lz.bp && x < c1 - c0) ? __ldg(Lz.bp + c0 + x) : 0.f;
    }
  };
  load_shares(p.layers[0]);
  const int wrp = wrow_bytes(WT, d) + 16;  // byte stride of a neuron item's rows
  const int rpn = gated ? 2 : 1;           // gate/up rows per neuron
  const int b1_off = (rpn + 1) * wrp;  // the b1 block, after the gate/up/down rows
  const int dn_off = rpn * wrp;        // the down row

  for (int l = 0; l < p.L; ++l) {
    const StackLayer& Ly = p.layers[l];
    const int r = Ly.rank;
    const int US = 2 * r + 16;  // byte stride of the fp16 u rows
    const int k0 = share_lo(r, c, G), k1 = share_lo(r, c + 1, G);
    if (t == 0) PI_STAMP(l, 0);
#pragma unroll
    for (int b = 0; b < B; ++b)
#pragma unroll
      for (int e = 0; e < EPT; ++e) y[b][e] = 0.f;
    float hsum[B];  // sum of the thread's token columns (Q4_0 dots)
#pragma unroll
    for (int b = 0; b < B; ++b) {
      hsum[b] = 0.f;
      if constexpr (WT == kQ4_0) {
#pragma unroll
        for (int e = 0; e < EPT; ++e) hsum[b] += h[b][e];
      }
    }

    // ---- predictor step 1: u = ReLU(P1 h) ----
    bool to = false;
    if constexpr (PT == kF16 && (B > 1 || kP1Mma)) {
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
          float psc = 1.f;
          if constexpr (PT == kQ4_0) {
            q4_codes<EPT>(s.ring + off, d, t, w, psc);  // same column ownership as Q4_0 weight rows
          } else {
            row_vals<WT, EPT, PT>(s.ring + off, t, T, w);
          }
          release_item();
#pragma unroll
          for (int b = 0; b < B; ++b) {
            float a = 0.f;
#pragma unroll
            for (int e = 0; e < EPT; ++e) a = fmaf(w[e], h[b][e], a);
            if constexpr (PT == kQ4_0) a = psc * fmaf(16.f, a, -24.f * hsum[b]);
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
    if (t == 0) PI_STAMP(l, 1);
#pragma unroll
    for (int i = 0; i < kShareRegs; ++i) {
      const int x = t + i * T;
      if (x < c1 - c0) s.bp[x] = bp_v[i];
    }
    // ---- neuron streams: groups of items until an end marker ----
    // Every warp takes the same barriers in the same order; a group's size is
    // read by thread 0 from the group's first item and passed on through
    // shared memory behind a barrier, so every warp agrees on it.
    float* gact = s.gred + kMaxGroup * (kMaxConsumers / 32) * 2 * B;  // [gs][B] activations
    auto head_size = [&](uint32_t it) -> int {  // thread 0 only
      to |= !mbar_wait(&s.full[it % kNQ], (it / kNQ) & 1u, ctrl);
      return to ? 0 : s.item_gs[it % kNQ];
    };
    auto run_stream = [&]() -> bool {
      if (t == 0) s.misc[2] = head_size(witem);
      if (named_sync_or(1, T, to)) return false;
      for (;;) {
        const int gs = s.misc[2];
        if (gs == 0) {  // the end marker: every warp releases it
          ++witem;
          release_item();
          return true;
        }
        for (int i = 0; i < gs; ++i) to |= !mbar_wait(&s.full[(witem + i) % kNQ], ((witem + i) / kNQ) & 1u, ctrl);
        if (!to) {
          if constexpr (WT == kF16 && PT == kF16 && kF16Mma) {
            // Tensor cores: the group's gate and up rows form one 16-row A tile
            // (unused rows repeat the first neuron), the fp16 token rows the B
            // tile; warps split d, partial dots meet in shared memory.
            const int bn = lane & 7;
            const uint32_t b_base =
                bn < B ? smem_u32(s.hb + bn * HS) + (uint32_t)(((lane >> 3) & 1) * 16) : smem_u32(s.zero);
            const uint32_t b_step = bn < B ? 32u : 0u;
            const int KS = d / 16, ks0 = warp * KS / NW, ks1 = (warp + 1) * KS / NW;
            const int tr = lane & 15;
            const int jj = tr / rpn < gs ? tr / rpn : 0;
            const int which = gated ? (tr & 1) : 0;  // item row: gate then up (ReGLU), up (otherwise)
            const uint32_t a_base = smem_u32(s.ring + s.item_off[(witem + jj) % kNQ]) + (uint32_t)(which * wrp) +
                                    (uint32_t)((lane >> 4) * 16);
            float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
            int ks = ks0;
            if (kMmaX2 && gs * rpn <= 8) {
              // rows 8-15 of the tile are unused: load rows 0-7 only (lanes 0-7
              // address k 0-7, lanes 8-15 k 8-15)
              const int tr8 = lane & 7;
              const int j8 = tr8 / rpn < gs ? tr8 / rpn : 0;
              const int w8 = gated ? (tr8 & 1) : 0;
              const uint32_t a8 = smem_u32(s.ring + s.item_off[(witem + j8) % kNQ]) + (uint32_t)(w8 * wrp) +
                                  (uint32_t)(((lane >> 3) & 1) * 16);
              for (; ks + 1 < ks1; ks += 2) {
                uint32_t a0, a2, b0, b1, e0, e2, f0, f1;
                ldsm_x2(a8 + 32u * ks, a0, a2);
                ldsm_x2(b_base + b_step * ks, b0, b1);
                ldsm_x2(a8 + 32u * (ks + 1), e0, e2);
                ldsm_x2(b_base + b_step * (ks + 1), f0, f1);
                mma_16816(acc0, a0, 0u, a2, 0u, b0, b1);
                mma_16816(acc1, e0, 0u, e2, 0u, f0, f1);
              }
            }
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
          } else {
            // CUDA cores: each thread's columns, the 2B dots of a neuron summed
            // over the warp together
            for (int jj = 0; jj < gs; ++jj) {
              const uint8_t* it = s.ring + s.item_off[(witem + jj) % kNQ];
              float acc[2 * B];
              // dots of the row at `at` with the thread's token columns
              auto dots = [&](const uint8_t* at, int base) {
                float wv[EPT];
                if constexpr (WT == kQ4_0) {
                  float sc;
                  q4_codes<EPT>(at, d, t, wv, sc);
#pragma unroll
                  for (int b = 0; b < B; ++b) {
                    float a = 0.f;
#pragma unroll
                    for (int e = 0; e < EPT; ++e) a = fmaf(wv[e], h[b][e], a);
                    acc[base + b] = sc * fmaf(16.f, a, -24.f * hsum[b]);
                  }
                } else {
                  w_vals<WT, EPT>(at, t, T, wv);
#pragma unroll
                  for (int b = 0; b < B; ++b) {
                    float a = 0.f;
#pragma unroll
                    for (int e = 0; e < EPT; ++e) a = fmaf(wv[e], h[b][e], a);
                    acc[base + b] = a;
                  }
                }
              };
              dots(it + (gated ? wrp : 0), B);
              if (gated) {
                dots(it, 0);
              } else {
#pragma unroll
                for (int b = 0; b < B; ++b) acc[b] = 0.f;
              }
              const float tot = warp_sums<2 * B>(acc, lane);
              if ((lane & (16 / B - 1)) == 0) s.gred[(jj * NW + warp) * 2 * B + lane / (16 / B)] = tot;
            }
          }
        }
        if (named_sync_or(1, T, to)) return false;  // every partial dot of the group is in
        if (t < gs * B) {
          const int jj = t / B, b = t % B;
          float gd = 0.f, vd = 0.f;
          if constexpr (WT == kF16 && PT == kF16 && kF16Mma) {
            for (int w = 0; w < NW; ++w) {
              gd += s.redp[w * 32 + (jj * rpn) * 2 + b];
              vd += s.redp[w * 32 + (jj * rpn + rpn - 1) * 2 + b];
            }
          } else {
            for (int w = 0; w < NW; ++w) {
              gd += s.gred[(jj * NW + w) * 2 * B + b];
              vd += s.gred[(jj * NW + w) * 2 * B + B + b];
            }
          }
          const uint32_t q = (witem + jj) % kNQ;
          const float bias =
              Ly.b1 ? reinterpret_cast<const float*>(s.ring + s.item_off[q] + b1_off)[s.item_j[q] & 3] : 0.f;
          gact[jj * B + b] = gated ? act_eval(kReglu, gd + bias, vd) : act_eval(p.act, vd + bias, 0.f);
        }
        if (t == 0) s.misc[2] = head_size(witem + gs);  // the next group (or the end marker)
        if (named_sync_or(1, T, to)) return false;
        for (int jj = 0; jj < gs; ++jj) {
          float wd[EPT];
          const uint8_t* at = s.ring + s.item_off[(witem + jj) % kNQ] + dn_off;
          if constexpr (WT == kQ4_0) {
            float sc;
            q4_codes<EPT>(at, d, t, wd, sc);
#pragma unroll
            for (int e = 0; e < EPT; ++e) wd[e] = fmaf(wd[e], 16.f, -24.f);  // q - 8, exact
#pragma unroll
            for (int b = 0; b < B; ++b) {
              const float a = gact[jj * B + b] * sc;
#pragma unroll
              for (int e = 0; e < EPT; ++e) y[b][e] = fmaf(a, wd[e], y[b][e]);
            }
          } else {
            w_vals<WT, EPT>(at, t, T, wd);
#pragma unroll
            for (int b = 0; b < B; ++b) {
              const float a = gact[jj * B + b];
#pragma unroll
              for (int e = 0; e < EPT; ++e) y[b][e] = fmaf(a, wd[e], y[b][e]);
            }
          }
        }
        witem += gs;
        for (int i = 0; i < gs; ++i) release_item();
      }
    };

    named_sync(1, T);
    if (t == 0) mbar_arrive(s.u_bar);  // the barrier warp arrives at barrier U
    // the static hot neurons need no predictor: they fill the wait for barrier U
    if (!run_stream()) return;
    if (t == 0) PI_STAMP(l, 2);
      {
      // barrier U has passed and u is staged (the barrier warp's signal)
      const bool okw = mbar_wait(s.u_ready, l & 1, ctrl);
      if (named_sync_or(1, T, !okw)) return;
    }
    if (t == 0) PI_STAMP(l, 3);
    // the other accumulator buffer is free now (its last readers passed barrier U)
    {
      float4* nxt = reinterpret_cast<float4*>(p.yacc) + (size_t)((l + 1) & 1) * ybuf4;
      const int z0 = share_lo(ybuf4, c, G), z1 = share_lo(ybuf4, c + 1, G);
      for (int i = z0 + t; i < z1; i += T) nxt[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }

    // ---- predictor step 2: scores of this CTA's cold rows ----
    if constexpr (PT == kF16) {
      // Tensor cores: 16-row tiles of P2 (one ring item each) against the u
      // rows (hi, lo per token).  Each tile's k-steps are cut into KQ parts
      // so that every warp has work; partial scores meet in shared memory.
      const int nrows = c1 - c0;
      const int ntile = (nrows + 15) / 16;
      const int bn = lane & 7;
      const uint32_t b_base = (bn < 2 * B ? smem_u32(s.ub + bn * US) + (uint32_t)(((lane >> 3) & 1) * 16) : smem_u32(s.zero));
      const uint32_t b_step = bn < 2 * B ? 32u : 0u;
      const int KS = r / 16;
      int KQ = ntile > 0 ? (2 * NW + ntile - 1) / ntile : 1;
      if (KQ > KS / 4) KQ = KS / 4;
      if (KQ > kMaxKQ) KQ = kMaxKQ;
      if (KQ < 1) KQ = 1;
      const int cap = p.seg_cap;  // rows per k-part slot of the partial scores
      int released = 0;  // P2 tiles this warp has released; a tile is released once the warp is past it
      for (int un = warp; un < ntile * KQ; un += NW) {
        const int it = un / KQ, kq = un % KQ;
        for (; released < it; ++released) release_item();
        const uint32_t myitem = witem + it;
        to |= !mbar_wait(&s.full[myitem % kNQ], (myitem / kNQ) & 1u, ctrl);
        if (to) continue;  // the tile is read only once it has landed
        const int rows = min(16, nrows - 16 * it);
        const int ar = lane & 15;
        const uint32_t a_base = smem_u32(s.ring + s.item_off[myitem % kNQ]) + (uint32_t)((ar < rows ? ar : 0) * US) +
                                (uint32_t)((lane >> 4) * 16);
        float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
        const int ke = (kq + 1) * KS / KQ;
        int ks = kq * KS / KQ;
        for (; ks + 1 < ke; ks += 2) {
          uint32_t a0, a1, a2, a3, b0, b1, e0, e1, e2, e3, f0, f1;
          ldsm_x4(a_base + 32u * ks, a0, a1, a2, a3);
          ldsm_x2(b_base + b_step * ks, b0, b1);
          ldsm_x4(a_base + 32u * (ks + 1), e0, e1, e2, e3);
          ldsm_x2(b_base + b_step * (ks + 1), f0, f1);
          mma_16816(acc0, a0, a1, a2, a3, b0, b1);
          mma_16816(acc1, e0, e1, e2, e3, f0, f1);
        }
        if (ks < ke) {
          uint32_t a0, a1, a2, a3, b0, b1;
          ldsm_x4(a_base + 32u * ks, a0, a1, a2, a3);
          ldsm_x2(b_base + b_step * ks, b0, b1);
          mma_16816(acc0, a0, a1, a2, a3, b0, b1);
        }
        // thread (g, t4): rows g and g+8, columns 2*t4 (hi) and 2*t4+1 (lo) = token t4;
        // each k-part has its own slot, summed in k-part order below, so the
        // scores do not depend on which warp finished first
        const int g = lane >> 2, t4 = lane & 3;
        if (t4 < B) {
          float* slot = s.sc + (size_t)kq * cap * B;
          if (g < rows) slot[(16 * it + g) * B + t4] = (acc0[0] + acc1[0]) + (acc0[1] + acc1[1]);
          if (g + 8 < rows) slot[(16 * it + g + 8) * B + t4] = (acc0[2] + acc1[2]) + (acc0[3] + acc1[3]);
        }
      }
      for (; released < ntile; ++released) release_item();
      if (named_sync_or(1, T, to)) return;  // every partial score is in
      for (int x = t; x < nrows; x += T) {
        bool on = false;
#pragma unroll
        for (int b = 0; b < B; ++b) {
          float sc = 0.f;
          for (int q = 0; q < KQ; ++q) sc += s.sc[((size_t)q * cap + x) * B + b];
          on |= (sc + s.bp[x]) > Ly.thr;
        }
        s.act[x] = on ? 1 : 0;
      }
      witem += ntile;
    } else if constexpr (PT == kQ4_0) {
      // Q4_0 P2 rows, one warp per row: lane m takes 32-element blocks m,
      // m + 32, ...; a code q is placed in the top mantissa bits of 1.0f
      // (f = 1 + q/16, exact), so a block's dot is s (16 sum(f u) - 24 sum(u))
      // with the block sums of u staged with u
      const int nblk = r / 32, US1 = nblk + 1, RS = 32 * US1;
      const float* usum = s.u + (size_t)B * (p.rank + 32);
      for (int cc = c0; cc < c1; cc += NW) {
        const int rows = min(NW, c1 - cc);
        uint32_t off;
        to |= !wait_item(off);
        if (warp < rows) {
          const uint8_t* qrow = s.ring + off + (size_t)warp * (r / 2);
          const uint8_t* srow = s.ring + off + (size_t)rows * (r / 2) + (size_t)warp * (r / 16);
          float acc[B];
#pragma unroll
          for (int b = 0; b < B; ++b) acc[b] = 0.f;
          for (int m = lane; m < nblk; m += 32) {
            const uint4 q = *reinterpret_cast<const uint4*>(qrow + 16 * m);
            const float bsc = half_bits_to_float(*reinterpret_cast<const uint16_t*>(srow + 2 * m));
            const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
            float dot[B];
#pragma unroll
            for (int b = 0; b < B; ++b) dot[b] = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint32_t byte = qw[w] >> (8 * kk);
                const float flo = __uint_as_float(0x3f800000u | ((byte & 0xfu) << 19));
                const float fhi = __uint_as_float(0x3f800000u | ((byte & 0xf0u) << 15));
                const int e = 4 * w + kk;  // element e (low nibble) and e + 16 (high nibble)
#pragma unroll
                for (int b = 0; b < B; ++b) {
                  dot[b] = fmaf(flo, s.u[(size_t)b * RS + e * US1 + m], dot[b]);
                  dot[b] = fmaf(fhi, s.u[(size_t)b * RS + (e + 16) * US1 + m], dot[b]);
                }
              }
#pragma unroll
            for (int b = 0; b < B; ++b) acc[b] = fmaf(bsc, fmaf(16.f, dot[b], -24.f * usum[b * nblk + m]), acc[b]);
          }
          bool on = false;
          const float bias = s.bp[cc - c0 + warp];
#pragma unroll
          for (int b = 0; b < B; ++b) on |= (warp_sum(acc[b]) + bias) > Ly.thr;
          if (lane == 0) s.act[cc - c0 + warp] = on ? 1 : 0;
        }
        release_item();
      }
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
    if (t == 0) PI_STAMP(l, 4);
    // local ascending list of this CTA's active cold rows (consumer warp 0):
    // to the producer through shared memory, and parked in this CTA's own
    // stretch of idx (compacted after the last layer) with its count
    if (warp == 0) {
      int cnt = 0;
      int32_t* park = p.idx ? p.idx + (int64_t)l * C + c0 : nullptr;
      for (int x0 = 0; x0 < c1 - c0; x0 += 32) {
        const int x = x0 + lane;
        const bool on = x < c1 - c0 && s.act[x];
        const unsigned m = __ballot_sync(0xffffffffu, on);
        if (on) {
          const int at = cnt + __popc(m & ((1u << lane) - 1u));
          s.cidx[at] = H + c0 + x;
          if (park) park[at] = H + c0 + x;
        }
        cnt += __popc(m);
      }
      if (lane == 0) {
        s.misc[0] = cnt;
        p.lcnt[l * G + c] = cnt;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(s.list_bar);
      if (lane == 0) PI_STAMP(l, 5);
    }

    // ---- the neuron stream: claimed hot chunks and this CTA's predicted cold rows ----
    if (!run_stream()) return;
    if (t == 0) PI_STAMP(l, 6);

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
    if (l + 1 < p.L) load_shares(p.layers[l + 1]);  // in flight across barrier Y and the glue
    named_sync(1, T);
    if (t == 0) PI_STAMP(l, 7);
    if (t == 0) grid_arrive(ctrl);
    {
      bool okw = true;
      if (t == 0) okw = grid_wait(ctrl, base, 2 * l + 1, G);
      if (named_sync_or(1, T, !okw)) return;
    }
    if (t == 0) PI_STAMP(l, 8);

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
        for (int e = 0; e < EPT; ++e) h[b][e] = round_to(HT, h[b][e] * inv);
      }
      if constexpr (kTokRows) {
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
          for (int b = 0; b < B; ++b) store_vals<WT, EPT, HT>(dst + (size_t)b * d * ep, t, T, h[b]);
        }
      }
    }
    if (t == 0) PI_STAMP(l, 9);
  }
  // ---- the ascending lists: every CTA moves its parked list of each layer
  // to its offset (the sum of the lower CTAs' counts); layers in chunks whose
  // lists fit in the ring, one grid barrier per chunk between reads and writes
  unsigned nbar = 2u * p.L;
  if (C > 0) {
    // every take of every layer is done (barrier Y): clear this CTA's share of
    // the handed-over slots, so that the next launch finds them zero
    for (int l = 0; l < p.L; ++l) {
      const int n = (int)ld_relaxed_u32(&ctrl->don_push[l]);
      for (int i = share_lo(n, c, G) + t; i < share_lo(n, c + 1, G); i += T) p.don[(size_t)l * C + i] = 0;
    }
  }
  if (C > 0 && p.idx) {
    int* keep = reinterpret_cast<int*>(s.ring);                                // [chunk layers][seg_cap]
    int* offs = reinterpret_cast<int*>(s.ring) + p.cmp_layers * p.seg_cap;    // [chunk layers][2]: offset, total
    for (int l0 = 0; l0 < p.L; l0 += p.cmp_layers) {
      const int l1 = min(p.L, l0 + p.cmp_layers);
      for (int l = l0 + warp; l < l1; l += NW) {  // one warp per layer: this CTA's offset and the total
        int below = 0, all = 0;
        for (int i = lane; i < G; i += 32) {
          const int v = __ldcg(p.lcnt + l * G + i);
          all += v;
          if (i < c) below += v;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          below += __shfl_xor_sync(0xffffffffu, below, o);
          all += __shfl_xor_sync(0xffffffffu, all, o);
        }
        if (lane == 0) {
          offs[2 * (l - l0)] = below;
          offs[2 * (l - l0) + 1] = all;
        }
      }
      for (int l = l0; l < l1; ++l) {
        const int n = __ldcg(p.lcnt + l * G + c);
        for (int i = t; i < n; i += T) keep[(l - l0) * p.seg_cap + i] = __ldcg(p.idx + (int64_t)l * C + c0 + i);
      }
      named_sync(1, T);
      if (t == 0) grid_arrive(ctrl);
      {
        bool okw = true;
        if (t == 0) okw = grid_wait(ctrl, base, nbar, G);
        if (named_sync_or(1, T, !okw)) return;
      }
      ++nbar;
      for (int l = l0; l < l1; ++l) {
        const int n = __ldcg(p.lcnt + l * G + c);
        const int o = offs[2 * (l - l0)];
        for (int i = t; i < n; i += T) p.idx[(int64_t)l * C + o + i] = keep[(l - l0) * p.seg_cap + i];
        if (c == 0 && t == 0) p.counts[l] = offs[2 * (l - l0) + 1];
      }
      named_sync(1, T);  // offs and keep are reused by the next chunk
    }
  } else if (c == 0) {
    for (int l = t; l < p.L; l += T) p.counts[l] = 0;
  }
  // every CTA has passed the last barrier, so every claim is done: reset the
  // claim counters and leave the barrier base for the next launch
  if (c == 0) {
    for (int l = t; l < p.L; l += T) {
      p.pool[l] = 0;
      ctrl->don_push[l] = 0;
      ctrl->don_take[l] = 0;
      ctrl->don_done[l] = 0;
    }
    if (t == 0) atomicExch(&ctrl->bar_base, base + nbar * (unsigned)G);
  }
}

template <int WT, int PT, int B, int EPT>
cudaError_t launch_t(const StackParams& p, int G, size_t smem, cudaStream_t st) {
  auto fn = k_stack<WT, PT, B, EPT>;
  // the dynamic shared-memory limit is a per-device attribute of the kernel:
  // set it once on every device that launches it (the first launch on a
  // device should come before any stream capture)
  static std::mutex mu;
  static bool configured[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!configured[dev]) {
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
      if (e != cudaSuccess) return e;
      configured[dev] = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(p.T + 64);  // producer warp, consumer warps, barrier warp
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

int stack_ept(int d) { return (kEptMin == 8 && d % 256 == 0 && d / 8 <= kMaxConsumers) ? 8 : 16; }

bool stack_supported(int wtype, int ptype, int d, int ffn, int n_hot, int rank, int B, int L) {
  if (B < 1 || B > 2) return false;
  if (L < 1 || L > kMaxLayers) return false;
  const bool combo = (wtype == kF16 && ptype == kF16) || (wtype == kQ4_0 && ptype == kF16) ||
                     (wtype == kF32 && ptype == kF32) || (wtype == kQ4_0 && ptype == kQ4_0);
  if (!combo) return false;
  const int ept = stack_ept(d);
  if (d % (32 * ept) != 0 || d / ept > kMaxConsumers) return false;
  if (wtype == kQ4_0 && d % 256 != 0) return false;
  if (rank % 8 != 0 || rank > kMaxRank) return false;
  if (!stack_rank_ok(ptype, rank)) return false;
  (void)ffn;
  (void)n_hot;
  return true;
}

size_t stack_smem_layout(StackParams& p, int ptype, int B, int G) {
  const int C = p.ffn - p.n_hot;
  const int share_cap = (C + G - 1) / G + 1;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 127) & ~(size_t)127;
    return (int)o;
  };
  // the ring first, everything else at the end of shared memory
  const size_t sizes[] = {
      sizeof(uint64_t) * (2 * kNQ + 3),                                        // bars
      sizeof(uint32_t) * 4 * kNQ,                                              // item offsets, starts, rows, groups
      ptype == kF32 ? sizeof(float) * (size_t)B * p.rank                       // u (fp32 predictors)
      : ptype == kQ4_0 ? sizeof(float) * (size_t)B * (p.rank + 32 + p.rank / 32)  // u block-transposed + block sums
                       : 0,
      sizeof(float) * share_cap,                                               // bp
      sizeof(int) * share_cap,                                                 // cidx
      (size_t)share_cap,                                                       // act
      sizeof(float) * share_cap * B * kMaxKQ,                                  // sc (one slot per k-part)
      sizeof(float) * 2 * (kMaxConsumers / 32) * 6 * B,                        // red
      sizeof(float) * (kMaxGroup * (kMaxConsumers / 32) * 2 * B + kMaxGroup * B),  // gred + group activations
      sizeof(int) * 4,                                                         // misc
      stack_token_rows(ptype, B) ? (size_t)B * (2 * p.d + 16) : 0,             // hb
      ptype == kF16 ? (size_t)2 * B * (2 * p.rank + 16) : 0,                   // ub (fp16 predictors)
      16,                                                                      // zero
      stack_token_rows(ptype, B) ? sizeof(float) * (kMaxConsumers / 32) * 32 : 0,  // redp
  };
  size_t fixed = 0;
  for (size_t b : sizes) fixed += (b + 127) & ~(size_t)127;
  const size_t total = kSmemBytes;
  if (fixed + 32768 > total) return 0;
  const size_t ring = (total - fixed) & ~(size_t)127;
  p.ring_bytes = (int)ring;
  p.seg_cap = share_cap;
  off = ring;
  p.off_bars = take(sizes[0]);
  p.off_itemoff = take(sizes[1]);
  p.off_u = take(sizes[2]);
  p.off_bp = take(sizes[3]);
  p.off_cidx = take(sizes[4]);
  p.off_act = take(sizes[5]);
  p.off_sc = take(sizes[6]);
  p.off_red = take(sizes[7]);
  p.off_gred = take(sizes[8]);
  p.off_misc = take(sizes[9]);
  p.off_hb = take(sizes[10]);
  p.off_ub = take(sizes[11]);
  p.off_zero = take(sizes[12]);
  p.off_redp = take(sizes[13]);
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
  PI_STACK_CASE(kQ4_0, kQ4_0, 1, 8)
  PI_STACK_CASE(kQ4_0, kQ4_0, 2, 8)
  PI_STACK_CASE(kQ4_0, kQ4_0, 1, 16)
  PI_STACK_CASE(kQ4_0, kQ4_0, 2, 16)
#undef PI_STACK_CASE
  return cudaErrorInvalidValue;
}

}  // namespace pi
