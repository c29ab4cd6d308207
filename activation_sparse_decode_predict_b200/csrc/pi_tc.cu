// pi_tc.cu -- the sparse FFN of a token block of 3..16 tokens on the fifth-
// generation tensor cores: tcgen05.mma with fp32 accumulators in tensor memory,
// operands gathered into shared memory by TMA (fp16 weights and tokens).
//
// PowerInfer (unite.ai, "Nöron Bilinçli Operatör"; aibars.net,
// "Sparsity-Nutzung"): only the rows of the hot neurons and of the
// predicted-active cold neurons are read.  With several tokens in a block each
// streamed row serves all of them, so the neuron-aware operator becomes a
// product of gathered tiles:
//
//   up    D[128 listed neurons x 16 tokens] = W_rows[128 x d] . h^T[d x 16]
//         (gate and up rows: two accumulators), tiles of 128 list positions
//   down  D[128 output columns x 32] = W_downT^T[128 x listed] . A^T[listed x 32]
//         where A holds each activation as an fp16 pair hi + lo (hi rows 0-15,
//         lo rows 16-31), so the product keeps ~22 bits of the fp32 activation.
//
// Gathers: a 2-D tensor map over a weight matrix with a one-row box of 64
// columns; tile::gather4 brings four arbitrary rows per instruction into a
// 128-byte-swizzled operand tile (the swizzle follows the shared-memory
// address, so a row may land at any row of an aligned 1024-byte atom).
//
// Work split, both kernels: a flat sequence of units (up: tile x 64-column
// block of d; down: 256-column chunk of d x 64-position block of the list) is
// cut into G contiguous ranges of equal length, one per CTA; a CTA accumulates
// consecutive units of the same tile (chunk) in tensor memory and writes one
// partial per (CTA, tile) segment.  The writers of a tile (chunk) follow from
// the same arithmetic; each counts itself on a per-tile (per-chunk) counter,
// and the last one to count sums the partials in CTA order -- the same sum
// whichever CTA is last: deterministic.
//
// Kernels per call: k_tc_up (gate/up dots; the last writer of a tile adds b1,
// applies the activation and writes the fp16 hi/lo rows) -> k_tc_down (down
// products; the last writer of a chunk adds b2 and writes y).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstring>
#include <mutex>

#include "pi_common.cuh"
#include "pi_launch.h"
#include "pi_sync.cuh"
#include "pi_tc.cuh"

namespace pi {

namespace {

#ifndef PI_TC_KBS
#define PI_TC_KBS 2
#endif
#ifndef PI_TC_CHUNK
#define PI_TC_CHUNK 256
#endif
// Warps 0-3 issue the TMA gathers, one warp per SM sub-partition: the
// gathers of one warp are issued lane after lane, and a single warp cannot
// issue them fast enough to keep HBM busy (about a third of the rate of four
// warps).  Warp 4 issues the MMAs and owns the tensor memory; warps 5-8 are
// the epilogue (warp w reads tensor-memory lanes 32 (w % 4) .. + 31).
#ifndef PI_TC_PW
#define PI_TC_PW 8
#endif
constexpr int kProdWarps = PI_TC_PW;
static_assert(kProdWarps == 2 || kProdWarps == 4 || kProdWarps == 8, "2, 4 or 8 producer warps");
constexpr int kMmaWarp = kProdWarps;
constexpr int kTcThreads = 32 * (kProdWarps + 5);
constexpr int kTcSlots = 8;         // up partials per tile at most
constexpr int kGMaxWriters = 296;   // CTAs of the largest grid: writers of a down chunk at most
constexpr int kSmemAvail = 227 * 1024 - 2048;  // stages fit below this (barriers + alignment slack after them)
// up: 64-column blocks of d per stage; each block is [gate 16 KB][up 16 KB][tokens 2 KB]
constexpr int kUpKBS = PI_TC_KBS;
constexpr int kUpBlock = 34 * 1024;
constexpr int kUpStage = kUpKBS * kUpBlock;
constexpr int kUpNS = kSmemAvail / kUpStage;
// down: output columns per chunk (kChunk / 128 products of M = 128); a stage is
// [kChunk/64 column blocks x 64 positions x 128 B][activations 32 x 128 B]
constexpr int kChunk = PI_TC_CHUNK;
constexpr int kDnCB = kChunk / 64;
constexpr int kDnStage = kDnCB * 8192 + 4096;
constexpr int kDnNS = kSmemAvail / kDnStage;
constexpr int kDnCols = 2 * 32 * (kChunk / 128);  // tensor-memory columns: two buffers x (kChunk/128) x N = 32
constexpr int kBarBytes = 1024;      // mbarriers and the tensor-memory address, after the stages
static_assert(kUpNS >= 3 && kDnNS >= 3, "at least three stages in flight");
static_assert(kChunk == 256 || kChunk == 512, "down chunks of 256 or 512 columns");

// ---------------------------------------------------------------------------
// the flat unit sequence and its split into contiguous per-CTA ranges

struct Split {
  int64_t U;  // units
  int G;      // CTAs that get a (non-empty) range
};

__device__ __forceinline__ int64_t range_lo(const Split& s, int c) { return s.U * c / s.G; }

// CTA whose range holds unit u (0 <= u < U)
__device__ __forceinline__ int range_owner(const Split& s, int64_t u) {
  int c = (int)((u * s.G) / s.U);
  while (c > 0 && range_lo(s, c) > u) --c;
  while (c + 1 < s.G && range_lo(s, c + 1) <= u) ++c;
  return c;
}

// the list length (hot rows + predicted) with the count clamped to [0, C]
__device__ __forceinline__ int list_total(const int32_t* count, int n_hot, int ffn, Ctrl* ctrl, bool report) {
  int cnt = __ldcg(count);
  const int C = ffn - n_hot;
  if (cnt < 0 || cnt > C) {
    if (report) set_status(&ctrl->status, kStCapacity);
    cnt = cnt < 0 ? 0 : C;
  }
  return n_hot + cnt;
}

// up: units = 128-position tiles x 64-column blocks of d; every range holds at
// least a quarter of a tile, so a tile has at most 5 writers
__device__ __forceinline__ Split up_split(int ntot, int d, int G) {
  const int KB = d / (64 * kUpKBS);
  Split s;
  s.U = (int64_t)((ntot + 127) / 128) * KB;
  const int64_t per = KB / 4 > 0 ? KB / 4 : 1;
  const int64_t g = s.U / per;
  s.G = g < G ? (g > 0 ? (int)g : 1) : G;
  return s;
}

// down: units = 256-column chunks of d x 64-position blocks of the list;
// d / 256 <= G, so a range spans at most two chunks
__device__ __forceinline__ Split down_split(int ntot, int d, int G) {
  const int KBp = (ntot + 63) / 64;
  Split s;
  s.U = (int64_t)(d / kChunk) * KBp;
  s.G = s.U < G ? (s.U > 0 ? (int)s.U : 1) : G;
  return s;
}

// storage row of list position pos (hot rows first); an entry outside
// [n_hot, ffn) is reported and replaced by row 0
__device__ __forceinline__ int list_row_at(int pos, int ntot, int n_hot, int ffn, const int32_t* idx, Ctrl* ctrl) {
  if (pos < n_hot) return pos;
  if (pos >= ntot) return 0;  // beyond the list: any valid row, its products are dropped or multiplied by zero
  const int j = __ldcg(idx + (pos - n_hot));
  if (j < n_hot || j >= ffn) {
    set_status(&ctrl->status, kStIndex);
    return 0;
  }
  return j;
}

// The same in two steps: the raw entry (a load that may still be in flight),
// then its check once the value is needed.
__device__ __forceinline__ int list_raw(int pos, int ntot, int n_hot, const int32_t* idx) {
  if (pos < n_hot) return pos;
  if (pos >= ntot) return 0;
  return __ldcg(idx + (pos - n_hot));
}
__device__ __forceinline__ int list_checked(int j, int pos, int ntot, int n_hot, int ffn, Ctrl* ctrl) {
  if (pos >= n_hot && pos < ntot && (j < n_hot || j >= ffn)) {
    set_status(&ctrl->status, kStIndex);
    return 0;
  }
  return j;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

// ---------------------------------------------------------------------------
// up: gate/up dots of 128-neuron tiles -> pre[slot][pos][2][16]

struct TcUpParams {
  CUtensorMap tm_h;   // token block [B, d] fp16; box 64 x 16 (rows past B read as zero)
  CUtensorMap tm_w0;  // gate rows (ReGLU) or up rows [F, d] fp16; box 64 x 1
  CUtensorMap tm_w1;  // up rows (ReGLU); box 64 x 1
  CUtensorMap tm_t0;  // the same two matrices with a box of 64 x 128: a tile of hot rows in one load
  CUtensorMap tm_t1;
  const int32_t* idx;
  const int32_t* count;
  float* pre;      // [kTcSlots][ffn][2][16] partial dots of tiles with several writers
  const float* b1;
  __half* act16;   // [32][fpad] activations as fp16 hi / lo rows
  int* tcnt;       // [tiles] writers counted so far (zero between calls)
  Ctrl* ctrl;
  int d, ffn, n_hot, gated, act, B, fpad;
};

__global__ void __launch_bounds__(kTcThreads, 1) k_tc_up(const __grid_constant__ TcUpParams p) {
  extern __shared__ uint8_t smraw[];
  __shared__ int s_last;  // set by the epilogue: this CTA finishes the tile
  pdl_trigger();
  pdl_wait();  // the list, its count and the token block come from the kernels before
  uint8_t* sm = align1024(smraw);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + kUpNS * kUpStage);
  uint64_t* empty = full + kUpNS;
  uint64_t* accf = empty + kUpNS;  // [2] accumulators ready
  uint64_t* acce = accf + 2;       // [2] accumulators drained
  uint64_t* done = acce + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  Ctrl* ctrl = p.ctrl;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const int ntot = list_total(p.count, p.n_hot, p.ffn, ctrl, c == 0 && threadIdx.x == 0);
  const int KB = p.d / (64 * kUpKBS);  // units per tile
  const Split sp = up_split(ntot, p.d, gridDim.x);
  const int64_t u0 = c < sp.G ? range_lo(sp, c) : 0, u1 = c < sp.G ? range_lo(sp, c + 1) : 0;
  const int nmat = p.gated ? 2 : 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kUpNS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], 4);
    }
    mbar_init(done, 1);
    mbar_fence_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tslot, 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp < kProdWarps) {
    // ---------------- TMA producers: a tile's 32 four-row groups are split
    // evenly over the producer warps; lane l < 2 gpw of warp w gathers group
    // g = w gpw + l % gpw from the gate (l < gpw) or up (l >= gpw) rows ----------------
    constexpr int gpw = 32 / kProdWarps;
    const int g = gpw * warp + lane % gpw, m = lane / gpw;
    const bool mine = m == 0 || (m == 1 && p.gated);
    int r[4] = {0, 0, 0, 0};
    int cur = -1;
    int64_t issued = 0;
    bool ok = true;
    // units: (tile, column block) pairs counted along the range without divisions
    int t_nx = (int)(u0 / KB), k_nx = (int)(u0 % KB);
    for (int64_t u = u0; u < u1 && ok; ++u) {
      const int it = (int)(u - u0), s = it % kUpNS;
      const int tile = t_nx, kb = k_nx;
      if (++k_nx == KB) { k_nx = 0; ++t_nx; }
      // a tile of hot rows only is 128 consecutive storage rows: one tiled load per matrix
      const bool hot_tile = tile * 128 + 128 <= p.n_hot;
      if (tile != cur) {
        cur = tile;
        if (mine && !hot_tile) {
#pragma unroll
          for (int i = 0; i < 4; ++i) r[i] = list_row_at(tile * 128 + 4 * g + i, ntot, p.n_hot, p.ffn, p.idx, ctrl);
        }
      }
      if (it >= kUpNS) ok = mbar_wait(&empty[s], ((it / kUpNS) - 1) & 1, ctrl);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      // the stage's byte count is posted once; copies of the other warps that
      // land first leave the count below zero until then, and the phase cannot
      // complete before this arrival
      if (warp == 0 && lane == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)(kUpKBS * (nmat * 16384 + 2048)));
      __syncwarp();
      // the unit's column blocks back to back, so that a row's pieces are requested together
#pragma unroll
      for (int k = 0; k < kUpKBS; ++k) {
        uint8_t* st = sm + s * kUpStage + k * kUpBlock;
        const int x = (kb * kUpKBS + k) * 64;
        if (hot_tile) {
          if (warp == 0 && lane < nmat) tma_load_2d(st + lane * 16384, lane ? &p.tm_t1 : &p.tm_t0, x, tile * 128, &full[s]);
        } else if (mine) {
          tma_gather4(st + m * 16384 + g * 512, m ? &p.tm_w1 : &p.tm_w0, x, r[0], r[1], r[2], r[3], &full[s]);
        }
        if (warp == kProdWarps - 1 && lane == 31) tma_load_2d(st + 32768, &p.tm_h, x, 0, &full[s]);
      }
      ++issued;
    }
    // the CTA leaves only once every issued stage has landed (every producer
    // warp's copies count toward the same phases)
    if (warp == 0 && lane == 0)
      for (int64_t it = issued > kUpNS ? issued - kUpNS : 0; it < issued; ++it)
        mbar_wait(&full[it % kUpNS], (uint32_t)((it / kUpNS) & 1), ctrl);
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(128, 16, 0, 0);
      int buf = 0, nseg = 0, cur = -1;
      bool ok = true;
      int t_nx = (int)(u0 / KB), k_nx = (int)(u0 % KB);
      for (int64_t u = u0; u < u1; ++u) {
        const int it = (int)(u - u0), s = it % kUpNS;
        const int tile = t_nx;
        if (++k_nx == KB) { k_nx = 0; ++t_nx; }
        const bool first = tile != cur;
        const bool last = (u + 1 == u1) || k_nx == 0;
        if (first) {
          cur = tile;
          // this accumulator buffer was last used two segments ago: wait until it is drained
          if (nseg >= 2) ok = mbar_wait(&acce[buf], (uint32_t)(((nseg - 2) / 2) & 1), ctrl);
        }
        if (ok) ok = mbar_wait(&full[s], (uint32_t)((it / kUpNS) & 1), ctrl);
        if (!ok) break;
        tc_fence_after();
        const uint32_t dg = tmem + (uint32_t)(buf * 32);
#pragma unroll
        for (int k = 0; k < kUpKBS; ++k) {
          const uint32_t st = smem_u32(sm + s * kUpStage + k * kUpBlock);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = sw128_desc(st + 32768 + kk * 32, 16, 1024);
            const uint32_t acc = (first && k == 0 && kk == 0) ? 0u : 1u;
            tc_mma_f16(dg, sw128_desc(st + kk * 32, 16, 1024), bd, idesc, acc);
            if (p.gated) tc_mma_f16(dg + 16, sw128_desc(st + 16384 + kk * 32, 16, 1024), bd, idesc, acc);
          }
        }
        tc_commit(&empty[s]);
        if (last) {
          tc_commit(&accf[buf]);
          buf ^= 1;
          ++nseg;
        }
      }
      // every MMA of this thread has completed before tensor memory is freed
      tc_commit(done);
      mbar_wait(done, 0, ctrl);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue: warp quarter q reads tensor-memory lanes 32q..32q+31 ----------------
    // A tile written by one CTA is finished from registers.  A tile split
    // between CTAs: each writer stores its partial dots in its slot and counts
    // itself; the last writer to count sums the slots in CTA order (the same
    // sum whoever is last) and finishes the tile.
    const int q = warp & 3, et = threadIdx.x - 32 * (kMmaWarp + 1);
    int buf = 0, nseg = 0;
    int t_nx = (int)(u0 / KB), k_nx = (int)(u0 % KB);
    for (int64_t u = u0; u < u1; ++u) {
      const int tile = t_nx;
      if (++k_nx == KB) { k_nx = 0; ++t_nx; }
      const bool last = (u + 1 == u1) || k_nx == 0;
      if (!last) continue;
      // the segment's bookkeeping and this position's bias are looked up while
      // the accumulators are still being filled
      const int pos = tile * 128 + q * 32 + lane;
      const int c_lo = range_owner(sp, (int64_t)tile * KB);
      const int nw = range_owner(sp, (int64_t)tile * KB + KB - 1) - c_lo + 1, slot = c - c_lo;
      // an entry outside [n_hot, ffn) (reported by the producers) adds nothing:
      // its activation is zero
      bool valid = false;
      float bias = 0.f;
      if (pos < ntot) {
        const int j = list_raw(pos, ntot, p.n_hot, p.idx);
        valid = pos < p.n_hot || (j >= p.n_hot && j < p.ffn);
        if (valid && p.b1) bias = __ldg(p.b1 + j);
      }
      const bool okw = mbar_wait(&accf[buf], (uint32_t)((nseg / 2) & 1), ctrl);
      if (named_sync_or(1, 128, !okw)) break;  // all epilogue warps leave together
      tc_fence_after();
      float g[16], v[16];
      const uint32_t ta = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * 32);
      tmem_ld16(ta, g);
      if (p.gated) {
        tmem_ld16(ta + 16, v);
      } else {
#pragma unroll
        for (int b = 0; b < 16; ++b) v[b] = 0.f;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[buf]);
      buf ^= 1;
      ++nseg;
      if (nw > 1) {
        if (slot >= kTcSlots) {
          if (et == 0) set_status(&ctrl->status, kStCapacity);
        } else if (pos < ntot) {
          float4* dst = reinterpret_cast<float4*>(p.pre + (((size_t)slot * p.ffn + pos) * 2) * 16);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_float4(g[4 * i], g[4 * i + 1], g[4 * i + 2], g[4 * i + 3]);
          if (p.gated) {
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[4 + i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          }
        }
        // the CTA barrier orders every epilogue thread's stores before thread 0's
        // fence and count (release); the last writer's thread 0 fences after
        // its count (acquire) before the barrier that lets the others read
        named_sync(1, 128);
        if (et == 0) {
          __threadfence();
          const int prev = atomicAdd(p.tcnt + tile, 1);
          s_last = prev == nw - 1;
          if (prev == nw - 1) {
            p.tcnt[tile] = 0;  // every writer has counted: ready for the next call
            __threadfence();
          }
        }
        named_sync(1, 128);
        if (!s_last) continue;
#pragma unroll
        for (int b = 0; b < 16; ++b) g[b] = v[b] = 0.f;
        if (pos < ntot) {
#pragma unroll
          for (int sl = 0; sl < kTcSlots; ++sl) {
            if (sl >= nw) break;
            const float4* src = reinterpret_cast<const float4*>(p.pre + (((size_t)sl * p.ffn + pos) * 2) * 16);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float4 x = __ldcg(src + i);
              g[4 * i] += x.x; g[4 * i + 1] += x.y; g[4 * i + 2] += x.z; g[4 * i + 3] += x.w;
            }
            if (p.gated) {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float4 x = __ldcg(src + 4 + i);
                v[4 * i] += x.x; v[4 * i + 1] += x.y; v[4 * i + 2] += x.z; v[4 * i + 3] += x.w;
              }
            }
          }
        }
      }
      // bias + activation; fp16 hi/lo rows of the down operand, zero for tokens
      // past B and for positions past the list up to the next 64
      if (pos < ((ntot + 63) & ~63) && pos < p.fpad) {
        float a[16];
#pragma unroll
        for (int b = 0; b < 16; ++b) a[b] = 0.f;
        if (valid) {
#pragma unroll
          for (int b = 0; b < 16; ++b)
            if (b < p.B) a[b] = p.gated ? act_eval(kReglu, g[b] + bias, v[b]) : act_eval(p.act, g[b] + bias, 0.f);
        }
#pragma unroll
        for (int b = 0; b < 16; ++b) {
          const __half hi = __float2half_rn(a[b]);
          const __half lo = __float2half_rn(a[b] - __half2float(hi));
          p.act16[(size_t)b * p.fpad + pos] = hi;
          p.act16[(size_t)(16 + b) * p.fpad + pos] = lo;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

// ---------------------------------------------------------------------------
// down: partial outputs of 256-column chunks -> part[cta][segment][16][256]

struct TcDownParams {
  CUtensorMap tm_wd;   // W_downT [F, d] fp16; box 64 x 1
  CUtensorMap tm_wdt;  // the same with a box of 64 x 64: a block of hot positions in one load per column block
  CUtensorMap tm_act;  // act16 [32, fpad] fp16; box 64 x 32
  const int32_t* idx;
  const int32_t* count;
  float* part;  // [G][2][16][kChunk]
  const float* b2;
  float* y;     // [B][d]
  int* ccnt;    // [d / kChunk] writers counted so far (zero between calls)
  Ctrl* ctrl;
  int d, ffn, n_hot, B;
};

__global__ void __launch_bounds__(kTcThreads, 1) k_tc_down(const __grid_constant__ TcDownParams p) {
  extern __shared__ uint8_t smraw[];
  __shared__ int s_last;  // set by the epilogue: this CTA finishes the chunk
  __shared__ int s_woff[kGMaxWriters];  // the chunk's partial outputs, by writer (offsets into part)
  pdl_trigger();
  pdl_wait();  // the list, its count and the activation rows come from the kernels before
  uint8_t* sm = align1024(smraw);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + kDnNS * kDnStage);
  uint64_t* empty = full + kDnNS;
  uint64_t* accf = empty + kDnNS;
  uint64_t* acce = accf + 2;
  uint64_t* done = acce + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  Ctrl* ctrl = p.ctrl;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const int ntot = list_total(p.count, p.n_hot, p.ffn, ctrl, false);
  const int KBp = (ntot + 63) / 64;
  const Split sp = down_split(ntot, p.d, gridDim.x);
  const int64_t u0 = c < sp.G ? range_lo(sp, c) : 0, u1 = c < sp.G ? range_lo(sp, c + 1) : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDnNS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], 4);
    }
    mbar_init(done, 1);
    mbar_fence_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tslot, kDnCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp < kProdWarps) {
    // ---------------- TMA producers: a unit's 16 x kDnCB four-position gathers
    // are split evenly over the producer warps; lane l < opw of warp w does
    // gather o = w opw + l: list positions 4 (o / kDnCB) .. + 3, column block
    // o % kDnCB (neighbouring lanes ask for neighbouring pieces of the same rows) ----------------
    constexpr int opw = kDnCB * 16 / kProdWarps;
    static_assert(opw <= 32, "one gather per lane and unit");
    const int o = opw * warp + lane, cbo = o % kDnCB, pg = o / kDnCB;
    const bool mine = lane < opw;
    int64_t issued = 0;
    bool ok = true;
    // the list entries of a unit are loaded two units ahead and checked when
    // the unit is issued, so that no lookup waits on the path from a free
    // stage to its copies
    int ra[4] = {0, 0, 0, 0}, rb[4] = {0, 0, 0, 0};
    // units: (chunk, position block) pairs counted along the range without
    // divisions; kb2 is the position block two units ahead
    int c_nx = KBp > 0 ? (int)(u0 / KBp) : 0, k_nx = KBp > 0 ? (int)(u0 % KBp) : 0;
    int kb2 = k_nx;
    if (mine) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (u0 < u1) ra[i] = list_raw(kb2 * 64 + 4 * pg + i, ntot, p.n_hot, p.idx);
      }
    }
    if (++kb2 == KBp) kb2 = 0;
    if (mine) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (u0 + 1 < u1) rb[i] = list_raw(kb2 * 64 + 4 * pg + i, ntot, p.n_hot, p.idx);
      }
    }
    for (int64_t u = u0; u < u1 && ok; ++u) {
      const int it = (int)(u - u0), s = it % kDnNS;
      const int chunk = c_nx, kb = k_nx;
      if (++k_nx == KBp) { k_nx = 0; ++c_nx; }
      if (++kb2 == KBp) kb2 = 0;
      int r[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        r[i] = ra[i];
        ra[i] = rb[i];
        if (mine && u + 2 < u1) rb[i] = list_raw(kb2 * 64 + 4 * pg + i, ntot, p.n_hot, p.idx);
      }
      if (it >= kDnNS) ok = mbar_wait(&empty[s], ((it / kDnNS) - 1) & 1, ctrl);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      if (warp == 0 && lane == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)(kDnCB * 8192 + 4096));
      __syncwarp();
      uint8_t* st = sm + s * kDnStage;
      if (mine) {
#pragma unroll
        for (int i = 0; i < 4; ++i) r[i] = list_checked(r[i], kb * 64 + 4 * pg + i, ntot, p.n_hot, p.ffn, ctrl);
      }
      if (kb * 64 + 64 <= p.n_hot) {
        // 64 hot positions are 64 consecutive storage rows
        if (warp == 0 && lane < kDnCB)
          tma_load_2d(st + lane * 8192, &p.tm_wdt, chunk * kChunk + lane * 64, kb * 64, &full[s]);
      } else if (mine) {
        tma_gather4(st + cbo * 8192 + 4 * pg * 128, &p.tm_wd, chunk * kChunk + cbo * 64, r[0], r[1], r[2], r[3],
                    &full[s]);
      }
      if (warp == kProdWarps - 1 && lane == 31) tma_load_2d(st + kDnCB * 8192, &p.tm_act, kb * 64, 0, &full[s]);
      ++issued;
    }
    if (warp == 0 && lane == 0)
      for (int64_t it = issued > kDnNS ? issued - kDnNS : 0; it < issued; ++it)
        mbar_wait(&full[it % kDnNS], (uint32_t)((it / kDnNS) & 1), ctrl);
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(128, 32, 1, 0);
      int buf = 0, nseg = 0, cur = -1;
      bool ok = true;
      int c_nx = KBp > 0 ? (int)(u0 / KBp) : 0, k_nx = KBp > 0 ? (int)(u0 % KBp) : 0;
      for (int64_t u = u0; u < u1; ++u) {
        const int it = (int)(u - u0), s = it % kDnNS;
        const int chunk = c_nx;
        if (++k_nx == KBp) { k_nx = 0; ++c_nx; }
        const bool first = chunk != cur;
        const bool last = (u + 1 == u1) || k_nx == 0;
        if (first) {
          cur = chunk;
          if (nseg >= 2) ok = mbar_wait(&acce[buf], (uint32_t)(((nseg - 2) / 2) & 1), ctrl);
        }
        if (ok) ok = mbar_wait(&full[s], (uint32_t)((it / kDnNS) & 1), ctrl);
        if (!ok) break;
        tc_fence_after();
        const uint32_t st = smem_u32(sm + s * kDnStage);
#pragma unroll
        for (int m = 0; m < kChunk / 128; ++m) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            // A: MN-major, 64-column blocks 8 KB apart, 8-position groups 1 KB apart;
            // k-step kk = positions 16kk..16kk+15
            const uint64_t ad = sw128_desc(st + (2 * m) * 8192 + kk * 2048, 8192, 1024);
            const uint64_t bd = sw128_desc(st + kDnCB * 8192 + kk * 32, 16, 1024);
            tc_mma_f16(tmem + (uint32_t)(buf * (kDnCols / 2) + m * 32), ad, bd, idesc, (first && kk == 0) ? 0u : 1u);
          }
        }
        tc_commit(&empty[s]);
        if (last) {
          tc_commit(&accf[buf]);
          buf ^= 1;
          ++nseg;
        }
      }
      tc_commit(done);
      mbar_wait(done, 0, ctrl);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue: partial outputs of the CTA's chunk segments;
    // the last writer of a chunk to count itself sums the chunk's partials in
    // CTA order, adds b2 and writes y ----------------
    const int q = warp & 3, et = threadIdx.x - 32 * (kMmaWarp + 1);
    if (KBp == 0 && c < p.d / kChunk) {
      // an empty list: y = b2 (CTA c writes chunk c)
      for (int i = et; i < p.B * kChunk; i += 128) {
        const int col = c * kChunk + i % kChunk;
        p.y[(size_t)(i / kChunk) * p.d + col] = p.b2 ? __ldg(p.b2 + col) : 0.f;
      }
    }
    int buf = 0, nseg = 0;
    int c_nx = KBp > 0 ? (int)(u0 / KBp) : 0, k_nx = KBp > 0 ? (int)(u0 % KBp) : 0;
    for (int64_t u = u0; u < u1; ++u) {
      const int chunk = c_nx;
      if (++k_nx == KBp) { k_nx = 0; ++c_nx; }
      const bool last = (u + 1 == u1) || k_nx == 0;
      if (!last) continue;
      const int c_lo = range_owner(sp, (int64_t)chunk * KBp);
      const int nw = range_owner(sp, (int64_t)chunk * KBp + KBp - 1) - c_lo + 1;
      const bool okw = mbar_wait(&accf[buf], (uint32_t)((nseg / 2) & 1), ctrl);
      if (named_sync_or(1, 128, !okw)) break;  // all epilogue warps leave together
      tc_fence_after();
      // segment 0: the chunk of this CTA's first unit; segment 1: the next one
      const int seg = (u0 / KBp == chunk) ? 0 : 1;
      float* dst = p.part + ((size_t)c * 2 + seg) * 16 * kChunk;
#pragma unroll
      for (int m = 0; m < kChunk / 128; ++m) {
        float hv[16], lv[16];
        const uint32_t ta = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * (kDnCols / 2) + m * 32);
        tmem_ld16(ta, hv);
        tmem_ld16(ta + 16, lv);
#pragma unroll
        for (int b = 0; b < 16; ++b)
          if (b < p.B) dst[b * kChunk + m * 128 + q * 32 + lane] = hv[b] + lv[b];  // token rows past B are not read
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[buf]);
      buf ^= 1;
      ++nseg;
      named_sync(1, 128);  // as in the up kernel: release by thread 0 after the barrier
      if (et == 0) {
        __threadfence();
        const int prev = atomicAdd(p.ccnt + chunk, 1);
        s_last = prev == nw - 1;
        if (prev == nw - 1) {
          p.ccnt[chunk] = 0;  // every writer has counted: ready for the next call
          __threadfence();
        }
      }
      named_sync(1, 128);
      if (!s_last) continue;
      for (int k = et; k < nw && k < kGMaxWriters; k += 128) {
        const int cw = c_lo + k;
        const int sg = (range_lo(sp, cw) / KBp == chunk) ? 0 : 1;
        s_woff[k] = (cw * 2 + sg) * 16 * kChunk;
      }
      named_sync(1, 128);
      // four columns per item and eight items per thread at once, so that the
      // loads of all of them are in flight together (this sum ends the kernel)
      const int nit = p.B * (kChunk / 4), nk = nw < kGMaxWriters ? nw : kGMaxWriters;
      for (int i0 = et; i0 < nit; i0 += 128 * 8) {
        float4 acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int i = i0 + 128 * j, col = chunk * kChunk + 4 * (i % (kChunk / 4));
          acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (i < nit && p.b2) acc[j] = make_float4(__ldg(p.b2 + col), __ldg(p.b2 + col + 1), __ldg(p.b2 + col + 2),
                                                    __ldg(p.b2 + col + 3));
        }
        for (int k = 0; k < nk; ++k) {
          const float* src = p.part + s_woff[k];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int i = i0 + 128 * j;
            if (i < nit) {
              const float4 x = __ldcg(reinterpret_cast<const float4*>(src + (i / (kChunk / 4)) * kChunk) + i % (kChunk / 4));
              acc[j].x += x.x; acc[j].y += x.y; acc[j].z += x.z; acc[j].w += x.w;
            }
          }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int i = i0 + 128 * j;
          if (i < nit) {
            float* dst = p.y + (size_t)(i / (kChunk / 4)) * p.d + chunk * kChunk + 4 * (i % (kChunk / 4));
            dst[0] = acc[j].x; dst[1] = acc[j].y; dst[2] = acc[j].z; dst[3] = acc[j].w;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kDnCols);
  }
}

// ---------------------------------------------------------------------------
// host: tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D fp16 tensor [rows, cols] (row pitch `pitch` bytes), box box_cols x box_rows, 128-byte swizzle
cudaError_t make_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t pitch, uint32_t box_cols,
                     uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;  // no driver entry point: the launch fails with PI_ERR_CUDA
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int tc_fpad(int ffn) { return (ffn + 63) & ~63; }

int tc_tiles(int ffn) { return (ffn + 127) / 128; }

// The token-block scratch: up partials, the activation rows, down partials and
// the per-tile / per-chunk writer counters (zero from pi_workspace_init on;
// each call leaves them at zero again).
struct TcScratch {
  float* pre;
  __half* act16;
  float* part;
  int* tcnt;
  int* ccnt;
};

size_t tc_align(size_t n) { return (n + 1023) & ~(size_t)1023; }

TcScratch tc_carve(void* scratch, int ffn) {
  TcScratch s;
  char* b = static_cast<char*>(scratch);
  s.pre = reinterpret_cast<float*>(b);
  b += tc_align((size_t)kTcSlots * ffn * 2 * 16 * 4);
  s.act16 = reinterpret_cast<__half*>(b);
  b += tc_align((size_t)32 * tc_fpad(ffn) * 2);
  s.part = reinterpret_cast<float*>(b);
  b += tc_align((size_t)296 * 2 * 16 * kChunk * 4);  // two segments per CTA
  s.tcnt = reinterpret_cast<int*>(b);
  b += tc_align((size_t)tc_tiles(ffn) * 4);
  s.ccnt = reinterpret_cast<int*>(b);
  return s;
}

}  // namespace

bool tc_ffn_supported(int wtype, int ptype, int d, int B) {
  if (wtype != kF16 || ptype != kF16) return false;
  if (B < 3 || B > 16) return false;
  return d % kChunk == 0 && d / kChunk <= 148;
}

size_t tc_ws_bytes(int d, int ffn, int B) {
  (void)d;
  (void)B;
  size_t n = tc_align((size_t)kTcSlots * ffn * 2 * 16 * 4);
  n += tc_align((size_t)32 * tc_fpad(ffn) * 2);
  n += tc_align((size_t)296 * 2 * 16 * kChunk * 4);
  n += tc_align((size_t)tc_tiles(ffn) * 4);
  n += tc_align((size_t)(148 + 1) * 4);  // chunk counters: d / kChunk <= 148
  return n;
}

cudaError_t launch_tc_ffn(int act, const void* h, int B, int d, int ffn, int n_hot, const int32_t* idx,
                          const int32_t* count, const void* wg, const void* wu, const void* wd, const float* b1,
                          const float* b2, float* y, void* scratch, Ctrl* ctrl, int sms, cudaStream_t st) {
  const int G = sms < 296 ? sms : 296;
  const int gated = act == kReglu;
  const TcScratch S = tc_carve(scratch, ffn);
  const int fpad = tc_fpad(ffn);
  cudaError_t e;

  TcUpParams U;
  memset(&U, 0, sizeof(U));
  if ((e = make_map(&U.tm_h, h, d, B, (uint64_t)d * 2, 64, 16)) != cudaSuccess) return e;
  if ((e = make_map(&U.tm_w0, gated ? wg : wu, d, ffn, (uint64_t)d * 2, 64, 1)) != cudaSuccess) return e;
  if ((e = make_map(&U.tm_w1, wu, d, ffn, (uint64_t)d * 2, 64, 1)) != cudaSuccess) return e;
  if ((e = make_map(&U.tm_t0, gated ? wg : wu, d, ffn, (uint64_t)d * 2, 64, 128)) != cudaSuccess) return e;
  if ((e = make_map(&U.tm_t1, wu, d, ffn, (uint64_t)d * 2, 64, 128)) != cudaSuccess) return e;
  U.idx = idx;
  U.count = count;
  U.pre = S.pre;
  U.b1 = b1;
  U.act16 = S.act16;
  U.tcnt = S.tcnt;
  U.ctrl = ctrl;
  U.d = d;
  U.ffn = ffn;
  U.n_hot = n_hot;
  U.gated = gated;
  U.act = act;
  U.B = B;
  U.fpad = fpad;
  const int up_smem = kUpNS * kUpStage + kBarBytes + 1024;
  if ((e = cudaFuncSetAttribute(k_tc_up, cudaFuncAttributeMaxDynamicSharedMemorySize, up_smem)) != cudaSuccess)
    return e;
  if ((e = launch_pdl(k_tc_up, dim3(G), dim3(kTcThreads), up_smem, st, U)) != cudaSuccess) return e;
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  TcDownParams D;
  memset(&D, 0, sizeof(D));
  if ((e = make_map(&D.tm_wd, wd, d, ffn, (uint64_t)d * 2, 64, 1)) != cudaSuccess) return e;
  if ((e = make_map(&D.tm_wdt, wd, d, ffn, (uint64_t)d * 2, 64, 64)) != cudaSuccess) return e;
  if ((e = make_map(&D.tm_act, S.act16, fpad, 32, (uint64_t)fpad * 2, 64, 32)) != cudaSuccess) return e;
  D.idx = idx;
  D.count = count;
  D.part = S.part;
  D.b2 = b2;
  D.y = y;
  D.ccnt = S.ccnt;
  D.ctrl = ctrl;
  D.d = d;
  D.ffn = ffn;
  D.n_hot = n_hot;
  D.B = B;
  const int dn_smem = kDnNS * kDnStage + kBarBytes + 1024;
  if ((e = cudaFuncSetAttribute(k_tc_down, cudaFuncAttributeMaxDynamicSharedMemorySize, dn_smem)) != cudaSuccess)
    return e;
  if ((e = launch_pdl(k_tc_down, dim3(G), dim3(kTcThreads), dn_smem, st, D)) != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace pi
