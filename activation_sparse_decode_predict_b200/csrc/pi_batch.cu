// pi_batch.cu -- the sparse FFN of a token block of 3..16 tokens on the
// tensor cores (fp16 tokens; fp16 weights, or Q4_0 gate/up rows whose codes
// are decoded in registers into the mma fragments).
//
// PowerInfer (unite.ai, "Nöron Bilinçli Operatör"; aibars.net,
// "Sparsity-Nutzung"): only the rows of the hot neurons and of the
// predicted-active cold neurons are read.  With several tokens in a block
// every streamed row serves all of them, so the per-neuron dots become small
// matrix products -- [rows x d] x [d x B] for gate/up and [B x n] x [n x d] for
// down -- done with mma.sync m16n8k16 (fp16 in, fp32 accumulate) while the
// weight rows stream through shared memory by 1-D bulk copies.  The work is
// HBM-bound (at most 16 FMAs per fp16 weight), so the tensor cores only have
// to keep up with the copies; the layout rules of the bulk copies and of
// ldmatrix decide the speed.
//
// k_rowdot CTA = (range of row positions, part of K).  16-row tiles of
//          weight rows (the FFN list's gate/up rows, or P1 / P2 rows) against
//          the token columns of the part: dots -> out[part][pos][slot][tok].
//          It also runs the predictor of a token block: P1 rows against the
//          tokens, then P2 rows against u split into fp16 hi + lo rows.
//          Q4_0 rows (list mode): codes and scales stream per row piece; the
//          codes become exact fp16 integers q - 8 in fragment order and each
//          block's scale multiplies its two k-steps' fp32 sums (the down
//          projection of Q4_0 blocks runs on the CUDA cores, pi_kernels_v1.cu).
// k_bdown  CTA = (chunk of d, range of list positions).  Activations from
//          pre (summed over the parts) and b1, split into fp16 hi + lo so the
//          product keeps ~22 bits of each activation; fp32 partial output of
//          the chunk -> partial[range][B][d]; the split-K reduce kernel adds
//          the ranges and b2.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "pi_batch.cuh"
#include "pi_common.cuh"
#include "pi_kernels_v1.cuh"
#include "pi_launch.h"
#include "pi_mma.cuh"
#include "pi_sync.cuh"

namespace pi {

namespace {

constexpr int kBW = 8;          // consumer warps
constexpr int kBT = kBW * 32;   // consumer threads
constexpr int kBSmem = 227 * 1024;
constexpr int kBMaxSlots = 8;
constexpr int kMapCap = 2048;  // list rows of a CTA's range kept in shared memory

__device__ __forceinline__ int bshare(int n, int c, int G) { return (int)((int64_t)n * c / G); }

// list position -> neuron row (hot rows first, then the predicted list);
// an entry outside [n_hot, ffn) is reported and replaced by row 0
__device__ __forceinline__ int list_row(int pos, int n_hot, int ffn, const int32_t* idx, Ctrl* ctrl) {
  if (pos < n_hot) return pos;
  const int j = __ldcg(idx + (pos - n_hot));
  if (j < n_hot || j >= ffn) {
    set_status(&ctrl->status, kStIndex);
    return -1;
  }
  return j;
}

// the rows of list positions n0.. (up to kMapCap of them) -> shared memory,
// loaded by the whole CTA at once; -1 marks an invalid list entry
__device__ __forceinline__ void load_rows(int* rmap, int n0, int n1, int n_hot, int ffn, const int32_t* idx,
                                          Ctrl* ctrl) {
  for (int i = threadIdx.x; i < n1 - n0 && i < kMapCap; i += blockDim.x) rmap[i] = list_row(n0 + i, n_hot, ffn, idx, ctrl);
}
__device__ __forceinline__ int row_at(const int* rmap, int pos, int n0, int n_hot, int ffn, const int32_t* idx,
                                      Ctrl* ctrl) {
  return pos - n0 < kMapCap ? rmap[pos - n0] : list_row(pos, n_hot, ffn, idx, ctrl);
}

__device__ __forceinline__ int clamp_count(const int32_t* count, int C, Ctrl* ctrl, bool report) {
  int cnt = __ldcg(count);
  if (cnt < 0 || cnt > C) {
    if (report) set_status(&ctrl->status, kStCapacity);
    cnt = cnt < 0 ? 0 : C;
  }
  return cnt;
}

// ---------------------------------------------------------------------------
// shared-memory layouts (host and device agree through these functions)

struct UpLayout {
  int PC, KC, HS, RS, SRS, SOFF, ISZ, off_map, off_h, off_red, off_ring, nslot, bytes;
};

// bytes of one 16-row slot of KC columns: fp16 rows, or Q4_0 rows as the
// KC / 2 code bytes then (SOFF on) the KC / 16 scale bytes of every row
__host__ __device__ inline int up_slot_bytes(int wt, int kc) {
  return wt == kQ4_0 ? 16 * (kc / 2 + 16) + 16 * (kc / 16 + 16) : 16 * (kc * 2 + 16);
}

__host__ __device__ inline UpLayout up_layout(int B8, int d, int S, int wt = kF16) {
  UpLayout L;
  L.PC = d / S;
  L.HS = L.PC * 2 + 16;   // token row stride (bytes): +16 keeps ldmatrix rows on distinct banks
  L.off_map = (2 * 8 * kBMaxSlots + 127) & ~127;
  L.off_h = L.off_map + kMapCap * 4;
  L.off_red = L.off_h + ((B8 * L.HS + 127) & ~127);
  L.off_ring = L.off_red + 2 * kBW * 16 * B8 * 4;
  const int room = kBSmem - L.off_ring;
  // columns per streamed chunk: the largest PC / m (a multiple of 16, at
  // most 2048; Q4_0: of 256, whole scale pieces, at most 4096) whose 16-row
  // slot leaves room for two slots -- fp16 row pieces of 4 KB in 64 KB slots
  // stream at full bandwidth, 2 KB pieces in 32 KB slots at about half of it,
  // even with more slots in flight
  const int step = wt == kQ4_0 ? 256 : 16, cap = wt == kQ4_0 ? 4096 : 2048;
  L.KC = step;
  for (int m = 1; m <= L.PC / step; ++m) {
    if (L.PC % m || (L.PC / m) % step || L.PC / m > cap) continue;
    if (2 * up_slot_bytes(wt, L.PC / m) <= room) {
      L.KC = L.PC / m;
      break;
    }
  }
  if (wt == kQ4_0) {
    L.RS = L.KC / 2 + 16;   // code row stride: rows start 4 banks apart
    L.SRS = L.KC / 16 + 16;
    L.SOFF = 16 * L.RS;
  } else {
    L.RS = L.KC * 2 + 16;   // weight row stride in a ring slot
    L.SRS = 0;
    L.SOFF = 0;
  }
  L.ISZ = up_slot_bytes(wt, L.KC);
  L.nslot = room / L.ISZ;
  if (L.nslot > kBMaxSlots) L.nslot = kBMaxSlots;
  L.bytes = L.off_ring + L.nslot * L.ISZ;
  return L;
}

struct DownLayout {
  int DCOLS, RS, ISZ, off_pre, off_b1, off_map, off_a, off_ring, nslot, bytes;
};

constexpr int kARow = 48;  // bytes per token row of an activation tile (16 fp16 + pad: conflict-free ldmatrix)

__host__ __device__ inline DownLayout down_layout(int d) {
  DownLayout L;
  // 4 KB row pieces where d allows (they stream at full bandwidth)
  L.DCOLS = (d % 2048 == 0) ? 2048 : (d % 1024 == 0) ? 1024 : (d % 512 == 0) ? 512 : 256;
  L.RS = L.DCOLS * 2 + 16;
  // a slot: the 16 W_downT row pieces, the tile's pre-activation block of
  // every part ([part][16][2][16] fp32 at most) and the 16-byte b1 blocks
  L.off_pre = 16 * L.RS;
  L.off_b1 = L.off_pre + 4 * 16 * 2 * 16 * 4;
  L.ISZ = L.off_b1 + 16 * 16;
  L.off_map = (2 * 8 * kBMaxSlots + 127) & ~127;
  L.off_a = L.off_map + kMapCap * 4;
  L.off_ring = L.off_a + 2 * 2 * 16 * kARow;  // [tile parity][hi, lo][16 token rows]
  L.off_ring = (L.off_ring + 127) & ~127;
  const int room = kBSmem - L.off_ring;
  L.nslot = room / L.ISZ;
  if (L.nslot > kBMaxSlots) L.nslot = kBMaxSlots;
  L.bytes = L.off_ring + L.nslot * L.ISZ;
  return L;
}

// ---------------------------------------------------------------------------

// Row dots against a block of token rows: out[part][pos][slot][tok] =
// sum over the part's columns of W[row(pos)] * x[tok].  List mode: positions
// are the FFN list [0, n_hot) ++ idx (gate and up rows of 8 neurons per
// 16-row tile when gated, else up rows of 16, slot 0 = gate, 1 = up); plain
// mode: rows 0..nrows-1 of one matrix, slot 0.
struct RowDotParams {
  const __half* x;   // [ntok, K] token rows
  const void* w0;    // gate (gated list mode) or the only matrix: fp16 rows, or Q4_0 codes
  const void* w1;    // up (gated list mode)
  const void* w0_sc;  // Q4_0 scales of w0 / w1 (list mode only)
  const void* w1_sc;
  const int32_t* idx;
  const int32_t* count;
  float* out;  // [S][R][W][ntok]
  Ctrl* ctrl;
  int ntok, K, S;
  int list;    // 1: FFN list mode
  int gated;   // list mode: gate and up rows
  int R;       // positions per part in out (ffn in list mode, nrows in plain mode)
  int nrows;   // plain mode
  int n_hot, ffn;
  int W;       // slots per position
  // token rows made on the fly (P2 of a token block): x row 2b = hi(u_b),
  // row 2b+1 = lo(u_b), u = ReLU(sum over upre_parts of upre [part][K][ntok/2])
  const float* upre;
  int upre_parts;
};

// Q4_0 rows (list mode): a lane's 4 code bytes 4t..4t+3 of a row's 32-column
// block, as the exact fp16 pairs (q - 8) of the block's k-step 0 (low
// nibbles: columns 4t, 4t+1 and 4t+2, 4t+3) and k-step 1 (high nibbles:
// the same + 16).  The token rows are staged in that column order, so the
// products pair up; each block's scale multiplies its two steps' sums in fp32.
__device__ __forceinline__ void q4_frag(uint32_t w, uint32_t& lo01, uint32_t& lo23, uint32_t& hi01, uint32_t& hi23) {
  const uint32_t p01 = __byte_perm(w, 0u, 0x4140), p23 = __byte_perm(w, 0u, 0x4342);
  const __half2 k1032 = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));  // 1024 + 8
  const __half2 k16th = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));  // 1 / 16
  const __half2 km72 = __halves2half2(__ushort_as_half(0xD480), __ushort_as_half(0xD480));   // -72
  auto h2 = [](uint32_t v) { return *reinterpret_cast<__half2*>(&v); };
  auto u32 = [](__half2 v) { return *reinterpret_cast<uint32_t*>(&v); };
  // (v | 0x6400) read as fp16 is 1024 + v for v < 1024: nibble q -> 1024 + q, high nibble -> 1024 + 16 q
  lo01 = u32(__hsub2(h2((p01 & 0x000F000Fu) | 0x64006400u), k1032));
  lo23 = u32(__hsub2(h2((p23 & 0x000F000Fu) | 0x64006400u), k1032));
  hi01 = u32(__hfma2(h2((p01 & 0x00F000F0u) | 0x64006400u), k16th, km72));
  hi23 = u32(__hfma2(h2((p23 & 0x00F000F0u) | 0x64006400u), k16th, km72));
}

template <int NT, int WT>
__global__ void __launch_bounds__(kBT + 32, 1) k_rowdot(const __grid_constant__ RowDotParams p) {
  static_assert(WT == kF16 || WT == kQ4_0, "fp16 or Q4_0 rows");
  extern __shared__ __align__(128) uint8_t sm[];
  const UpLayout Lay = up_layout(NT * 8, p.K, p.S, WT);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm);
  uint64_t* empty = full + kBMaxSlots;
  int* rmap = reinterpret_cast<int*>(sm + Lay.off_map);
  uint8_t* hs = sm + Lay.off_h;
  float* red = reinterpret_cast<float*>(sm + Lay.off_red);
  uint8_t* ring = sm + Lay.off_ring;
  Ctrl* ctrl = p.ctrl;

  pdl_trigger();
  // list mode: the rows to stream come from the kernels before; plain mode
  // streams rows that no kernel writes, so the producer starts before the
  // previous kernel has finished and only the consumers wait (for the token rows)
  if (p.list) pdl_wait();
  const int R = gridDim.x / p.S;
  const int rho = blockIdx.x / p.S, sig = blockIdx.x % p.S;
  const int col0 = sig * Lay.PC;
  const int ntot = p.list ? p.n_hot + clamp_count(p.count, p.ffn - p.n_hot, ctrl, blockIdx.x == 0 && threadIdx.x == 0)
                          : p.nrows;
  const int two = p.list && p.gated;  // two rows (gate, up) per position
  const int npt = two ? 8 : 16;       // positions per 16-row tile
  // whole tiles per range: only the last tile of the list is partial
  const int tall = (ntot + npt - 1) / npt;
  const int n0 = min(ntot, npt * bshare(tall, rho, R)), n1 = min(ntot, npt * bshare(tall, rho + 1, R));
  const int ntile = (n1 - n0 + npt - 1) / npt;
  const int nch = Lay.PC / Lay.KC;
  const int nitems = ntile * nch;
  const int nslot = Lay.nslot;

  if (threadIdx.x == 0) {
    for (int q = 0; q < nslot; ++q) {
      mbar_init(&full[q], 1);
      mbar_init(&empty[q], kBW);
    }
    mbar_fence_init();
  }
  if (p.list) load_rows(rmap, n0, n1, p.n_hot, p.ffn, p.idx, ctrl);
  __syncthreads();

  if (threadIdx.x < 32) {
    // ---------------- producer warp: one row per lane ----------------
    const int lane = threadIdx.x;
    for (int it = 0; it < nitems; ++it) {
      const int q = it % nslot;
      bool ok = true;
      if (it >= nslot) ok = mbar_wait(&empty[q], ((it / nslot) - 1) & 1, ctrl);
      if (!__all_sync(0xffffffffu, ok)) return;
      const int tile = it / nch, ch = it % nch;
      if constexpr (WT == kQ4_0) {
        // lanes 0-15: the rows' code pieces; lanes 16-31: their scale pieces
        if (lane == 0) mbar_arrive_expect_tx(&full[q], 16u * (uint32_t)(Lay.KC / 2 + Lay.KC / 16));
        __syncwarp();
        const int r16 = lane & 15;
        int pos = n0 + tile * npt + (two ? r16 / 2 : r16);
        if (pos >= n1) pos = n1 - 1;  // tail rows repeat the last one; their dots are dropped
        int j = row_at(rmap, pos, n0, p.n_hot, p.ffn, p.idx, ctrl);
        if (j < 0) j = 0;
        const bool up = two && (r16 & 1);
        const int64_t c0 = col0 + (int64_t)ch * Lay.KC;
        if (lane < 16)
          bulk_g2s(ring + q * Lay.ISZ + r16 * Lay.RS,
                   static_cast<const uint8_t*>(up ? p.w1 : p.w0) + (int64_t)j * (p.K / 2) + c0 / 2, Lay.KC / 2u,
                   &full[q]);
        else
          bulk_g2s(ring + q * Lay.ISZ + Lay.SOFF + r16 * Lay.SRS,
                   static_cast<const uint8_t*>(up ? p.w1_sc : p.w0_sc) + (int64_t)j * (p.K / 16) + c0 / 16,
                   Lay.KC / 16u, &full[q]);
      } else {
        if (lane == 0) mbar_arrive_expect_tx(&full[q], 16u * Lay.KC * 2u);
        __syncwarp();
        if (lane < 16) {
          int pos = n0 + tile * npt + (two ? lane / 2 : lane);
          if (pos >= n1) pos = n1 - 1;  // tail rows repeat the last one; their dots are dropped
          int j = p.list ? row_at(rmap, pos, n0, p.n_hot, p.ffn, p.idx, ctrl) : pos;
          if (j < 0) j = 0;
          const __half* mat = static_cast<const __half*>((two && (lane & 1)) ? p.w1 : p.w0);
          bulk_g2s(ring + q * Lay.ISZ + lane * Lay.RS, mat + (int64_t)j * p.K + col0 + ch * Lay.KC, Lay.KC * 2u,
                   &full[q]);
        }
      }
      __syncwarp();
    }
    // the CTA may exit only once its copies have landed
    for (int it = nitems > nslot ? nitems - nslot : 0; it < nitems; ++it)
      if (lane == 0) mbar_wait(&full[it % nslot], (it / nslot) & 1, ctrl);
    return;
  }

  // ---------------- consumer warps ----------------
  if (!p.list) pdl_wait();
  const int t = threadIdx.x - 32, cw = t >> 5, lane = t & 31;
  // this part's token columns -> shared memory (rows >= ntok are zero)
  if (p.upre) {
    // rows made from u: every upre value of the part is loaded once, with
    // 16-byte loads that are all in flight together
    const int nb = p.ntok / 2;
    const int nvec = Lay.PC * nb / 4;  // float4s of one part of upre
    for (int i0 = t; i0 < nvec; i0 += 4 * kBT) {
      float4 a[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) a[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int sp = 0; sp < p.upre_parts; ++sp) {
        const float4* src = reinterpret_cast<const float4*>(p.upre + ((int64_t)sp * p.K + col0) * nb);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int i = i0 + k * kBT;
          if (i < nvec) {
            const float4 v = __ldcg(src + i);
            a[k].x += v.x; a[k].y += v.y; a[k].z += v.z; a[k].w += v.w;
          }
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int i = i0 + k * kBT;
        if (i < nvec) {
          const float f[4] = {a[k].x, a[k].y, a[k].z, a[k].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int el = 4 * i + e, col = el / nb, tb = el % nb;
            const float u = fmaxf(f[e], 0.f);
            const __half hi = __float2half_rn(u);
            const __half lo = __float2half_rn(u - __half2float(hi));
            reinterpret_cast<__half*>(hs + (2 * tb) * Lay.HS)[col] = hi;
            reinterpret_cast<__half*>(hs + (2 * tb + 1) * Lay.HS)[col] = lo;
          }
        }
      }
    }
    const int units = Lay.PC / 8;
    for (int i = t; i < (NT * 8 - p.ntok) * units; i += kBT) {
      const int b = p.ntok + i / units, u = i % units;
      *reinterpret_cast<uint4*>(hs + b * Lay.HS + 16 * u) = make_uint4(0u, 0u, 0u, 0u);
    }
  } else {
    const int units = Lay.PC / 8;
    for (int i = t; i < NT * 8 * units; i += kBT) {
      const int b = i / units, u = i % units;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (b < p.ntok) v = __ldcg(reinterpret_cast<const uint4*>(p.x + (int64_t)b * p.K + col0) + u);
      if constexpr (WT == kQ4_0) {
        // column pairs in the order of q4_frag: within each 16 columns, pair w
        // goes to pair 4 (w % 2) + w / 2
        uint32_t* dst = reinterpret_cast<uint32_t*>(hs + b * Lay.HS + 32 * (u >> 1));
        const int h = 2 * (u & 1);
        dst[h] = v.x;
        dst[4 + h] = v.y;
        dst[h + 1] = v.z;
        dst[5 + h] = v.w;
      } else {
        *reinterpret_cast<uint4*>(hs + b * Lay.HS + 16 * u) = v;
      }
    }
  }
  named_sync(1, kBT);

  const int KSc = Lay.KC / 16;
  const int ks0 = cw * KSc / kBW, ks1 = (cw + 1) * KSc / kBW;
  const uint32_t a_lane = (uint32_t)((lane & 15) * Lay.RS + (lane >> 4) * 16);
  const uint32_t b_lane = smem_u32(hs) + (uint32_t)((lane & 7) * Lay.HS + ((lane >> 3) & 1) * 16);
  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
  bool to = false;
  for (int it = 0; it < nitems; ++it) {
    const int q = it % nslot;
    const int tile = it / nch, ch = it % nch;
    to |= !mbar_wait(&full[q], (it / nslot) & 1, ctrl);
    if (!to && WT == kQ4_0) {
      // this warp's 32-column blocks of the slot (KC / 32 is a multiple of 8)
      const int nblk = Lay.KC / 32, kb0 = cw * (nblk / kBW), kb1 = kb0 + nblk / kBW;
      const int g = lane >> 2, t4 = lane & 3;
      const uint8_t* slot = ring + q * Lay.ISZ;
      const uint8_t* cg = slot + g * Lay.RS + 4 * t4;
      const uint8_t* cg8 = cg + 8 * Lay.RS;
      const __half* sg = reinterpret_cast<const __half*>(slot + Lay.SOFF + g * Lay.SRS);
      const __half* sg8 = reinterpret_cast<const __half*>(slot + Lay.SOFF + (g + 8) * Lay.SRS);
      const uint32_t b_base = b_lane + (uint32_t)(ch * Lay.KC * 2);
      for (int kb = kb0; kb < kb1; ++kb) {
        uint32_t a0, a2, e0, e2, a1, a3, e1, e3;  // a: k-step 2 kb (low nibbles), e: 2 kb + 1 (high)
        q4_frag(*reinterpret_cast<const uint32_t*>(cg + 16 * kb), a0, a2, e0, e2);
        q4_frag(*reinterpret_cast<const uint32_t*>(cg8 + 16 * kb), a1, a3, e1, e3);
        const float s0 = __half2float(sg[kb]), s8 = __half2float(sg8[kb]);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          uint32_t b0, b1, f0, f1;
          ldsm_x2(b_base + (uint32_t)(nt * 8 * Lay.HS) + 64u * kb, b0, b1);
          ldsm_x2(b_base + (uint32_t)(nt * 8 * Lay.HS) + 64u * kb + 32u, f0, f1);
          float d4[4] = {0.f, 0.f, 0.f, 0.f};
          mma_16816(d4, a0, a1, a2, a3, b0, b1);
          mma_16816(d4, e0, e1, e2, e3, f0, f1);
          acc[nt][0] = fmaf(s0, d4[0], acc[nt][0]);
          acc[nt][1] = fmaf(s0, d4[1], acc[nt][1]);
          acc[nt][2] = fmaf(s8, d4[2], acc[nt][2]);
          acc[nt][3] = fmaf(s8, d4[3], acc[nt][3]);
        }
      }
    } else if (!to) {
      const uint32_t a_base = smem_u32(ring + q * Lay.ISZ) + a_lane;
      const uint32_t b_base = b_lane + (uint32_t)(ch * Lay.KC * 2);
      for (int ks = ks0; ks < ks1; ++ks) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(a_base + 32u * ks, a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          uint32_t b0, b1;
          ldsm_x2(b_base + (uint32_t)(nt * 8 * Lay.HS) + 32u * ks, b0, b1);
          mma_16816(acc[nt], a0, a1, a2, a3, b0, b1);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[q]);
    if (ch == nch - 1) {
      // tile complete: partial dots of each warp -> shared memory, summed per (row, token)
      constexpr int kRC = NT * 8;  // token columns of the reduction buffer
      float* rb = red + (tile & 1) * kBW * 16 * kRC;
      {
        const int g = lane >> 2, c2 = 2 * (lane & 3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float* w = rb + cw * 16 * kRC;
          w[g * kRC + nt * 8 + c2] = acc[nt][0];
          w[g * kRC + nt * 8 + c2 + 1] = acc[nt][1];
          w[(g + 8) * kRC + nt * 8 + c2] = acc[nt][2];
          w[(g + 8) * kRC + nt * 8 + c2 + 1] = acc[nt][3];
          acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
        }
      }
      if (named_sync_or(1, kBT, to)) return;
      for (int e = t; e < 16 * p.ntok; e += kBT) {
        const int row = e / p.ntok, tok = e % p.ntok;
        const int pos = n0 + tile * npt + (two ? row / 2 : row);
        if (pos < n1) {
          float v = 0.f;
#pragma unroll
          for (int w = 0; w < kBW; ++w) v += rb[(w * 16 + row) * kRC + tok];
          const int slot = two ? (row & 1) : p.W - 1;
          p.out[(((int64_t)sig * p.R + pos) * p.W + slot) * p.ntok + tok] = v;
        }
      }
    }
  }
}

// score = sum over the parts of (hi + lo dots) + bp; active = OR over the
// tokens of score > thr; one CTA per 256-row tile: 8 ballot words + count
// (the tile format of the compaction kernel).
__global__ void __launch_bounds__(256) k_bthresh(const float* sc, int S, int C, int B,
                                                 const float* __restrict__ bp, float thr,
                                                 uint32_t* __restrict__ tile_mask, int* __restrict__ tile_count) {
  __shared__ int cnt[8];
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x * 256 + threadIdx.x;
  bool on = false;
  if (c < C) {
    // the row's (hi, lo) dot pairs of each part are contiguous: one 8-byte
    // load per token, all in flight together
    const float bias = bp ? __ldg(bp + c) : 0.f;
    float v[16];
#pragma unroll
    for (int b = 0; b < 16; ++b) v[b] = 0.f;
    for (int s = 0; s < S; ++s) {
      const float2* q = reinterpret_cast<const float2*>(sc + ((int64_t)s * C + c) * 2 * B);
      float2 x[16];
#pragma unroll
      for (int b = 0; b < 16; ++b)
        if (b < B) x[b] = __ldcg(q + b);
#pragma unroll
      for (int b = 0; b < 16; ++b)
        if (b < B) v[b] += x[b].x + x[b].y;
    }
#pragma unroll
    for (int b = 0; b < 16; ++b) on |= b < B && (v[b] + bias) > thr;
  }
  const unsigned m = __ballot_sync(0xffffffffu, on);
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

struct BDownParams {
  const float* pre;   // [S][F][2][B]
  const float* b1;    // [F] or null
  const __half* wd;   // [F, d] (W_down transposed: neuron-major)
  const int32_t* idx;
  const int32_t* count;
  float* partial;     // [NR][B][d]
  Ctrl* ctrl;
  int B, d, ffn, n_hot, S, act, NR;
  int R;              // positions per part of pre (ffn + 16 spare, so that a 16-position block never runs past it)
};

template <int NT>
__global__ void __launch_bounds__(kBT + 32, 1) k_bdown(const __grid_constant__ BDownParams p) {
  extern __shared__ __align__(128) uint8_t sm[];
  const DownLayout Lay = down_layout(p.d);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm);
  uint64_t* empty = full + kBMaxSlots;
  int* rmap = reinterpret_cast<int*>(sm + Lay.off_map);
  uint8_t* abuf = sm + Lay.off_a;
  uint8_t* ring = sm + Lay.off_ring;
  Ctrl* ctrl = p.ctrl;
  pdl_trigger();
  pdl_wait();  // the list, its count and the pre-activations come from the kernels before

  const int DC = p.d / Lay.DCOLS;
  const int chi = blockIdx.x % DC, rho = blockIdx.x / DC;
  const int cbase = chi * Lay.DCOLS;
  const int C = p.ffn - p.n_hot;
  const int ntot = p.n_hot + clamp_count(p.count, C, ctrl, false);
  const int tall = (ntot + 15) / 16;  // whole 16-neuron tiles per range
  const int n0 = min(ntot, 16 * bshare(tall, rho, p.NR)), n1 = min(ntot, 16 * bshare(tall, rho + 1, p.NR));
  const int ntile = (n1 - n0 + 15) / 16;
  const int nslot = Lay.nslot;

  if (threadIdx.x == 0) {
    for (int q = 0; q < nslot; ++q) {
      mbar_init(&full[q], 1);
      mbar_init(&empty[q], kBW);
    }
    mbar_fence_init();
  }
  // activation tiles start zero (token rows >= B stay zero)
  for (int i = threadIdx.x; i < 2 * 2 * 16 * kARow / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(abuf)[i] = make_uint4(0u, 0u, 0u, 0u);
  load_rows(rmap, n0, n1, p.n_hot, p.ffn, p.idx, ctrl);
  __syncthreads();

  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    for (int it = 0; it < ntile; ++it) {
      const int q = it % nslot;
      bool ok = true;
      if (it >= nslot) ok = mbar_wait(&empty[q], ((it / nslot) - 1) & 1, ctrl);
      if (!__all_sync(0xffffffffu, ok)) return;
      const uint32_t preb = 16u * 2u * p.B * 4u;  // one part's pre-activation block of the tile
      if (lane == 0)
        mbar_arrive_expect_tx(&full[q], 16u * Lay.DCOLS * 2u + p.S * preb + (p.b1 ? 16u * 16u : 0u));
      __syncwarp();
      uint8_t* slot = ring + q * Lay.ISZ;
      if (lane < 16) {
        int pos = n0 + it * 16 + lane;
        if (pos >= n1) pos = n1 - 1;  // tail rows repeat the last one; their activations are zero
        int j = row_at(rmap, pos, n0, p.n_hot, p.ffn, p.idx, ctrl);
        if (j < 0) j = 0;
        bulk_g2s(slot + lane * Lay.RS, p.wd + (int64_t)j * p.d + cbase, Lay.DCOLS * 2u, &full[q]);
        if (p.b1) bulk_g2s(slot + Lay.off_b1 + 16 * lane, p.b1 + (j & ~3), 16u, &full[q]);
      } else if (lane < 16 + p.S) {
        // pre-activations of positions n0 + 16 it .. +15 (pre has 16 spare positions)
        const int sp = lane - 16;
        bulk_g2s(slot + Lay.off_pre + sp * preb, p.pre + (((int64_t)sp * p.R + n0 + it * 16) * 2) * p.B, preb,
                 &full[q]);
      }
      __syncwarp();
    }
    for (int it = ntile > nslot ? ntile - nslot : 0; it < ntile; ++it)
      if (lane == 0) mbar_wait(&full[it % nslot], (it / nslot) & 1, ctrl);
    return;
  }

  const int t = threadIdx.x - 32, cw = t >> 5, lane = t & 31;
  constexpr int kMT = 16;  // m-tiles (16 columns each) per warp at most
  const int MT = Lay.DCOLS / (kBW * 16);
  const int wcol = cw * MT * 16;  // this warp's first column within the chunk
  float acc[kMT][NT][4];
#pragma unroll
  for (int m = 0; m < kMT; ++m)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[m][nt][0] = acc[m][nt][1] = acc[m][nt][2] = acc[m][nt][3] = 0.f;
  const int gated = p.act == kReglu;
  const uint32_t a_lane = (uint32_t)(((lane & 7) + 8 * (lane >> 4)) * Lay.RS + ((lane >> 3) & 1) * 16 + wcol * 2);
  const uint32_t b_lane = smem_u32(abuf) + (uint32_t)((lane & 7) * kARow + ((lane >> 3) & 1) * 16);
  bool to = false;
  for (int it = 0; it < ntile; ++it) {
    const int q = it % nslot;
    const int buf = it & 1;
    const uint8_t* slot = ring + q * Lay.ISZ;
    to |= !mbar_wait(&full[q], (it / nslot) & 1, ctrl);
    // activations of the tile's 16 neurons from the slot, split into fp16 hi + lo
    if (!to && t < 16 * p.B) {
      const int i = t / p.B, b = t % p.B;
      const int pos = n0 + it * 16 + i;
      float a = 0.f;
      if (pos < n1) {
        const int j = row_at(rmap, pos, n0, p.n_hot, p.ffn, p.idx, ctrl);
        if (j >= 0) {
          float g = 0.f, v = 0.f;
          for (int sp = 0; sp < p.S; ++sp) {
            const float* pr = reinterpret_cast<const float*>(slot + Lay.off_pre) + (sp * 16 + i) * 2 * p.B;
            g += pr[b];
            v += pr[p.B + b];
          }
          const float bias = p.b1 ? reinterpret_cast<const float*>(slot + Lay.off_b1 + 16 * i)[j & 3] : 0.f;
          a = gated ? act_eval(kReglu, g + bias, v) : act_eval(p.act, v + bias, 0.f);
        }
      }
      const __half hi = __float2half_rn(a);
      const __half lo = __float2half_rn(a - __half2float(hi));
      reinterpret_cast<__half*>(abuf + ((buf * 2 + 0) * 16 + b) * kARow)[i] = hi;
      reinterpret_cast<__half*>(abuf + ((buf * 2 + 1) * 16 + b) * kARow)[i] = lo;
    }
    if (named_sync_or(1, kBT, to)) return;  // the tile's activations are in shared memory
    {
      const uint32_t a_base = smem_u32(ring + q * Lay.ISZ) + a_lane;
      uint32_t bh[NT][2], bl[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        ldsm_x2(b_lane + (uint32_t)(((buf * 2 + 0) * 16 + nt * 8) * kARow), bh[nt][0], bh[nt][1]);
        ldsm_x2(b_lane + (uint32_t)(((buf * 2 + 1) * 16 + nt * 8) * kARow), bl[nt][0], bl[nt][1]);
      }
#pragma unroll
      for (int m = 0; m < kMT; ++m) {
        if (m < MT) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(a_base + 32u * m, a0, a1, a2, a3);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            mma_16816(acc[m][nt], a0, a1, a2, a3, bh[nt][0], bh[nt][1]);
            mma_16816(acc[m][nt], a0, a1, a2, a3, bl[nt][0], bl[nt][1]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[q]);
  }
  if (named_sync_or(1, kBT, to)) return;
  // partial output of this range and chunk (zeros for an empty range)
  {
    const int g = lane >> 2, c2 = 2 * (lane & 3);
    float* out = p.partial + (int64_t)rho * p.B * p.d + cbase + wcol;
#pragma unroll
    for (int m = 0; m < kMT; ++m) {
      if (m < MT) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int b0 = nt * 8 + c2;
          if (b0 < p.B) {
            out[(int64_t)b0 * p.d + m * 16 + g] = acc[m][nt][0];
            out[(int64_t)b0 * p.d + m * 16 + g + 8] = acc[m][nt][2];
          }
          if (b0 + 1 < p.B) {
            out[(int64_t)(b0 + 1) * p.d + m * 16 + g] = acc[m][nt][1];
            out[(int64_t)(b0 + 1) * p.d + m * 16 + g + 8] = acc[m][nt][3];
          }
        }
      }
    }
  }
}

// n-tiles of 8 token rows the row-dot kernel stages (1, 2 or 4)
int rowdot_nt(int ntok) { return ntok <= 8 ? 1 : (ntok <= 16 ? 2 : 4); }

// parts of K such that the staged token columns of one part stay within
// 64 KB of shared memory

int row_parts(int ntok, int K) {
  const size_t bytes = (size_t)(8 * rowdot_nt(ntok)) * K * 2;
  int S = 1;
  while ((size_t)S * 65536 < bytes) S *= 2;
  return S;
}

template <int NT, int WT>
cudaError_t launch_rowdot_t(const RowDotParams& P, int G, cudaStream_t st) {
  const UpLayout UL = up_layout(NT * 8, P.K, P.S, WT);
  cudaError_t e = cudaFuncSetAttribute(k_rowdot<NT, WT>, cudaFuncAttributeMaxDynamicSharedMemorySize, UL.bytes);
  if (e != cudaSuccess) return e;
  e = launch_pdl(k_rowdot<NT, WT>, dim3(G), dim3(kBT + 32), UL.bytes, st, P);
  return e != cudaSuccess ? e : cudaGetLastError();
}

// wt: kF16 rows, or Q4_0 rows (list mode only)
cudaError_t launch_rowdot(const RowDotParams& P, int wt, int sms, cudaStream_t st) {
  const int G = (sms / P.S) * P.S;
  const int NT = rowdot_nt(P.ntok);
  if (wt == kQ4_0) {
    if (!P.list) return cudaErrorInvalidValue;
    if (NT == 1) return launch_rowdot_t<1, kQ4_0>(P, G, st);
    if (NT == 2) return launch_rowdot_t<2, kQ4_0>(P, G, st);
    return launch_rowdot_t<4, kQ4_0>(P, G, st);
  }
  if (NT == 1) return launch_rowdot_t<1, kF16>(P, G, st);
  if (NT == 2) return launch_rowdot_t<2, kF16>(P, G, st);
  return launch_rowdot_t<4, kF16>(P, G, st);
}

bool rowdot_fits(int ntok, int K, int wt = kF16) {
  const int S = row_parts(ntok, K);
  if (S > 4 || K % ((wt == kQ4_0 ? 256 : 128) * S) != 0) return false;
  return up_layout(8 * rowdot_nt(ntok), K, S, wt).nslot >= 2;  // the token tile the kernel stages
}

}  // namespace

bool batch_supported(int wtype, int htype, int d, int B) {
  if (htype != kF16 || B < kBatchMin || B > 16 || d % 256 != 0) return false;
  if (wtype == kF16) return rowdot_fits(B, d) && down_layout(d).nslot >= 2;
  if (wtype == kQ4_0) return rowdot_fits(B, d, kQ4_0);
  return false;
}

bool batch_pred_supported(int ptype, int d, int r, int B) {
  if (ptype != kF16 || B < kBatchMin || B > 16) return false;
  return rowdot_fits(B, d) && rowdot_fits(2 * B, r);
}

// positions per part of the pre-activation buffer: 16 spare (even, so that
// every 16-position block of any part starts on a 16-byte boundary)
int pre_positions(int ffn) { return (ffn + 16 + 1) & ~1; }

size_t batch_pre_bytes(int ffn, int B) { return (size_t)4 * pre_positions(ffn) * 2 * B * sizeof(float); }

int batch_ranges(int d, int sms) {
  const DownLayout D = down_layout(d);
  const int DC = d / D.DCOLS;
  const int NR = sms / DC;
  return NR < 1 ? 1 : NR;
}

cudaError_t launch_batch_predict(const void* h, int B, int d, int r, int C, int n_hot, const void* P1,
                                 const void* P2, const float* bp, float thr, float* upre, float* sc,
                                 uint32_t* tile_mask, int* tile_count, Ctrl* ctrl, int sms, cudaStream_t st) {
  RowDotParams U{};
  U.x = static_cast<const __half*>(h);
  U.w0 = static_cast<const __half*>(P1);
  U.out = upre;
  U.ctrl = ctrl;
  U.ntok = B;
  U.K = d;
  U.S = row_parts(B, d);
  U.R = r;
  U.nrows = r;
  U.W = 1;
  cudaError_t e = launch_rowdot(U, kF16, sms, st);
  if (e != cudaSuccess || C == 0) return e;
  RowDotParams S{};
  S.upre = upre;  // u = ReLU(sum of the P1 parts), split into hi + lo rows while staging
  S.upre_parts = U.S;
  S.w0 = static_cast<const __half*>(P2);
  S.out = sc;
  S.ctrl = ctrl;
  S.ntok = 2 * B;
  S.K = r;
  S.S = row_parts(2 * B, r);
  S.R = C;
  S.nrows = C;
  S.W = 1;
  e = launch_rowdot(S, kF16, sms, st);
  if (e != cudaSuccess) return e;
  e = launch_pdl(k_bthresh, dim3((C + 255) / 256), dim3(256), 0, st, static_cast<const float*>(sc), S.S, C, B, bp, thr,
                 tile_mask, tile_count);
  if (e != cudaSuccess) return e;
  (void)n_hot;
  return cudaGetLastError();
}

cudaError_t launch_batch_ffn(int act, int wtype, const void* h, int B, int d, int ffn, int n_hot, const int32_t* idx,
                             const int32_t* count, const void* wg, const void* wg_sc, const void* wu,
                             const void* wu_sc, const void* wd, const void* wd_sc, const float* b1, float* pre,
                             float* partial, int NR, Ctrl* ctrl, int sms, cudaStream_t st) {
  const int gated = act == kReglu;
  RowDotParams U{};
  U.x = static_cast<const __half*>(h);
  U.w0 = gated ? wg : wu;
  U.w1 = wu;
  U.w0_sc = gated ? wg_sc : wu_sc;
  U.w1_sc = wu_sc;
  U.idx = idx;
  U.count = count;
  U.out = pre;
  U.ctrl = ctrl;
  U.ntok = B;
  U.K = d;
  U.S = row_parts(B, d);
  U.list = 1;
  U.gated = gated;
  U.R = pre_positions(ffn);
  U.n_hot = n_hot;
  U.ffn = ffn;
  U.W = 2;
  cudaError_t e = launch_rowdot(U, wtype, sms, st);
  if (e != cudaSuccess) return e;
  if (wtype == kQ4_0)  // down on the CUDA cores, activations from the dots of every part
    return launch_ffn_down(kQ4_0, B, d, ffn, n_hot, idx, count, wd, wd_sc, nullptr, 0, partial, NR, st, pre, U.S, U.R,
                           b1, act);

  const int NT = B > 8 ? 2 : 1;
  BDownParams D;
  D.pre = pre;
  D.b1 = b1;
  D.wd = static_cast<const __half*>(wd);
  D.idx = idx;
  D.count = count;
  D.partial = partial;
  D.ctrl = ctrl;
  D.B = B;
  D.d = d;
  D.ffn = ffn;
  D.n_hot = n_hot;
  D.S = U.S;
  D.act = act;
  D.NR = NR;
  D.R = U.R;
  const DownLayout DL = down_layout(d);
  const int Gd = NR * (d / DL.DCOLS);
  if (NT == 1) {
    e = cudaFuncSetAttribute(k_bdown<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, DL.bytes);
    if (e != cudaSuccess) return e;
    e = launch_pdl(k_bdown<1>, dim3(Gd), dim3(kBT + 32), DL.bytes, st, D);
    if (e != cudaSuccess) return e;
  } else {
    e = cudaFuncSetAttribute(k_bdown<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, DL.bytes);
    if (e != cudaSuccess) return e;
    e = launch_pdl(k_bdown<2>, dim3(Gd), dim3(kBT + 32), DL.bytes, st, D);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace pi
