// pi_common.cuh -- element access, reductions and the device status word shared
// by the libpi kernels (sm_100a).
//
// Element types: fp32 and fp16 rows are read in 16-byte units (4 or 8
// elements); Q4_0 rows (split planes qs [rows, d/2] bytes, sc [rows, d/32]
// fp16) are read in 8-byte half-blocks of qs (16 elements) plus the block's
// fp16 scale.  In each 32-element block, byte k holds element k in its low
// nibble and element k + 16 in its high nibble; x = s * (q - 8) (GeekNews
// "Serving model bahasa besar ...", "Kuantisasi dan kompatibilitas": INT4
// Q4_0 with 32-element blocks and an fp16 scale).
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace pi {

enum : int { kF32 = 0, kF16 = 1, kQ4_0 = 2 };
enum : int { kRelu = 0, kReglu = 1, kRelu2 = 2 };

// Device status codes (same values as pi_status in pi.h).
enum : int { kStOk = 0, kStCapacity = -4, kStTimeout = -5, kStIndex = -6 };

// Workspace control block (first 256 bytes of every workspace).
struct Ctrl {
  int status;          // sticky: first device error wins
  int abort;           // set when any CTA of a persistent kernel gives up a wait
  int pad0[30];
  unsigned bar_count;  // grid barrier arrivals, monotonic (own 64-byte line)
  unsigned pad1[15];
  unsigned bar_base;   // bar_count at the start of the next persistent launch
  unsigned pad2[15];
  int pool[128];       // per-layer claim counters of the persistent kernel (zero between launches)
  unsigned don_push[128];  // per layer: cold rows handed to other CTAs (reserved slots)
  unsigned don_take[128];  // per layer: tickets taken on those slots
  unsigned don_done[128];  // per layer: CTAs that have decided what to hand over
};
static_assert(sizeof(Ctrl) == 2304, "control block is 2304 bytes");

__device__ __forceinline__ void set_status(int* status, int code) { atomicCAS(status, 0, code); }

// Programmatic dependent launch (kernels launched with launch_pdl): a kernel
// lets the next kernel on its stream be scheduled before it ends
// (pdl_trigger), and a thread waits for the previous kernel to complete with
// its memory visible (pdl_wait) before it reads anything that kernel wrote
// or writes global memory.  Work that depends on neither (barrier set-up,
// copies of weights nobody writes) may come before the wait.  Both are
// no-ops for a kernel launched without the attribute.  A kernel launched this
// way overlaps the previous one, so data that kernel writes is not read-only
// for this kernel's lifetime: it is read with plain or .cg loads after the
// wait, never through __ldg / const __restrict__ (the non-coherent read-only
// path, which the compiler may also move above the wait).
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Elements per access unit.
template <int T> struct Unit;
template <> struct Unit<kF32> { static constexpr int E = 4; };
template <> struct Unit<kF16> { static constexpr int E = 8; };
template <> struct Unit<kQ4_0> { static constexpr int E = 16; };

// Position (column) of the k-th element of unit u.
template <int T>
__device__ __forceinline__ int unit_col(int u, int k) {
  if constexpr (T == kQ4_0) {
    const int blk = u >> 1, half = u & 1;
    return blk * 32 + (k < 8 ? half * 8 + k : 16 + half * 8 + (k - 8));
  } else {
    return u * Unit<T>::E + k;
  }
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint2 ld_nc_v2(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}

__device__ __forceinline__ float2 h2f2(uint32_t v) {
  __half2 h = *reinterpret_cast<__half2*>(&v);
  return __half22float2(h);
}

__device__ __forceinline__ float half_bits_to_float(uint16_t v) {
  return __half2float(*reinterpret_cast<__half*>(&v));
}

// The raw bytes of unit u of row `row` of a [rows, d] matrix of type T
// (Q4_0: the 8 code bytes and the block's fp16 scale), and their decoding to
// floats.  Weights are streamed once, so loads bypass L1; a kernel that
// wants several units in flight loads them all before decoding any.
template <int T> struct WRaw { uint4 v; };
template <> struct WRaw<kQ4_0> { uint2 q; uint16_t s; };

template <int T>
__device__ __forceinline__ WRaw<T> load_w_raw(const void* __restrict__ data, const void* __restrict__ scales,
                                              int64_t row, int d, int u) {
  WRaw<T> r;
  if constexpr (T == kF32) {
    r.v = ld_nc_v4(reinterpret_cast<const float*>(data) + row * d + u * 4);
  } else if constexpr (T == kF16) {
    r.v = ld_nc_v4(reinterpret_cast<const __half*>(data) + row * d + u * 8);
  } else {
    r.q = ld_nc_v2(reinterpret_cast<const uint8_t*>(data) + row * (d / 2) + u * 8);
    r.s = __ldg(reinterpret_cast<const uint16_t*>(scales) + row * (d / 32) + (u >> 1));
  }
  return r;
}

template <int T>
__device__ __forceinline__ void decode_w(const WRaw<T>& r, float (&w)[Unit<T>::E]) {
  if constexpr (T == kF32) {
    w[0] = __uint_as_float(r.v.x); w[1] = __uint_as_float(r.v.y); w[2] = __uint_as_float(r.v.z); w[3] = __uint_as_float(r.v.w);
  } else if constexpr (T == kF16) {
    float2 f;
    f = h2f2(r.v.x); w[0] = f.x; w[1] = f.y;
    f = h2f2(r.v.y); w[2] = f.x; w[3] = f.y;
    f = h2f2(r.v.z); w[4] = f.x; w[5] = f.y;
    f = h2f2(r.v.w); w[6] = f.x; w[7] = f.y;
  } else {
    const float s = half_bits_to_float(r.s);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t b0 = (r.q.x >> (8 * k)) & 0xffu, b1 = (r.q.y >> (8 * k)) & 0xffu;
      w[k] = s * (float)((int)(b0 & 15u) - 8);
      w[4 + k] = s * (float)((int)(b1 & 15u) - 8);
      w[8 + k] = s * (float)((int)(b0 >> 4) - 8);
      w[12 + k] = s * (float)((int)(b1 >> 4) - 8);
    }
  }
}

// Load unit u of row `row` of a [rows, d] matrix of type T, decoded to floats.
template <int T>
__device__ __forceinline__ void load_w_unit(const void* __restrict__ data, const void* __restrict__ scales, int64_t row,
                                            int d, int u, float (&w)[Unit<T>::E]) {
  decode_w<T>(load_w_raw<T>(data, scales, row, d, u), w);
}

// Token values at the columns of unit u (layout of weight type WT) for token
// row `b` of h [*, ld] of type HT (kF32 or kF16).  Read-only cached loads
// (h is reused by every warp of a CTA), so the kernels that call this are
// launched without the dependent-launch attribute (see pdl_wait).
template <int WT, int HT>
__device__ __forceinline__ void load_h_unit(const void* __restrict__ h, int b, int ld, int u,
                                            float (&x)[Unit<WT>::E]) {
  constexpr int E = Unit<WT>::E;
  if constexpr (HT == kF32) {
    const float* hp = reinterpret_cast<const float*>(h) + (int64_t)b * ld;
    if constexpr (WT == kQ4_0) {
      const int c0 = unit_col<WT>(u, 0), c1 = unit_col<WT>(u, 8);
#pragma unroll
      for (int k = 0; k < 8; k += 4) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(hp + c0 + k));
        const float4 c = __ldg(reinterpret_cast<const float4*>(hp + c1 + k));
        x[k] = a.x; x[k + 1] = a.y; x[k + 2] = a.z; x[k + 3] = a.w;
        x[8 + k] = c.x; x[9 + k] = c.y; x[10 + k] = c.z; x[11 + k] = c.w;
      }
    } else {
#pragma unroll
      for (int k = 0; k < E; k += 4) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(hp + u * E + k));
        x[k] = a.x; x[k + 1] = a.y; x[k + 2] = a.z; x[k + 3] = a.w;
      }
    }
  } else {
    const __half* hp = reinterpret_cast<const __half*>(h) + (int64_t)b * ld;
    auto ld8 = [&](int col, float* o) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(hp + col));
      float2 f;
      f = h2f2(v.x); o[0] = f.x; o[1] = f.y;
      f = h2f2(v.y); o[2] = f.x; o[3] = f.y;
      f = h2f2(v.z); o[4] = f.x; o[5] = f.y;
      f = h2f2(v.w); o[6] = f.x; o[7] = f.y;
    };
    if constexpr (WT == kQ4_0) {
      ld8(unit_col<WT>(u, 0), x);
      ld8(unit_col<WT>(u, 8), x + 8);
    } else if constexpr (WT == kF16) {
      ld8(u * 8, x);
    } else {  // fp32 weights with fp16 tokens: 4 elements
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(hp + u * 4));
      float2 f = h2f2(v.x); x[0] = f.x; x[1] = f.y;
      f = h2f2(v.y); x[2] = f.x; x[3] = f.y;
    }
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// The activation with the kind chosen at run time (g: gate or up
// pre-activation incl. bias; v: up dot, used by ReGLU only).
__device__ __forceinline__ float act_eval(int act, float g, float v) {
  if (act == kReglu) return fmaxf(g, 0.f) * v;
  const float r = fmaxf(g, 0.f);
  return act == kRelu2 ? r * r : r;
}

template <int ACT>
__device__ __forceinline__ float activation(float g, float v) {
  if constexpr (ACT == kReglu) {
    return fmaxf(g, 0.f) * v;
  } else if constexpr (ACT == kRelu2) {
    const float r = fmaxf(g, 0.f);
    return r * r;
  } else {
    return fmaxf(g, 0.f);
  }
}

}  // namespace pi
