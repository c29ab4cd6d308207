// pi_tc.cuh -- fifth-generation tensor cores (tcgen05, accumulators in tensor
// memory) and TMA tensor loads for sm_100a, as one-instruction wrappers, plus
// the launcher of the token-block sparse FFN built on them (pi_tc.cu).
//
// Every load here is a plain tensor load into this CTA's shared memory: no
// cluster multicast anywhere.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "pi_common.cuh"
#include "pi_sync.cuh"

namespace pi {

// ---------------------------------------------------------------------------
// tensor memory

// Allocate `ncols` (a power of two, >= 32) columns of tensor memory for this
// CTA; the address lands in shared memory at `dst`.  One whole warp executes it.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 lanes x 16 columns of 32 bits from tensor memory (lane = the warp's quarter
// base + lane id), and the wait for the load, in one statement so that no use
// of the values can move above the wait.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// ---------------------------------------------------------------------------
// tcgen05.mma, kind::f16 (fp16 x fp16 -> fp32), A and B from shared memory

// Shared-memory matrix descriptor of a 128-byte-swizzled operand (sm_100
// layout: start address, leading and stride byte offsets in 16-byte units,
// version 1, swizzle mode 2 = 128 B).  K-major: rows of 128 bytes, 8-row
// groups `sbo` apart (lbo unused).  MN-major: 64-element blocks `lbo` apart,
// 8-row groups of k `sbo` apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor of kind::f16 with fp16 A and B, fp32 D: M x N, A/B
// K-major (0) or MN-major (1).
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A * B; issued by one thread.
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// ---------------------------------------------------------------------------
// TMA tensor loads into this CTA's shared memory (completion on an mbarrier)

// Box of a 2-D tensor map at (x, y); x must be a multiple of 16 bytes' worth of elements.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tm, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_u32(dst)),
      "l"(tm), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Four rows r0..r3 (any order, any rows) of a 2-D tensor map whose box is one
// row high, columns from x: they land as four consecutive box rows at dst.
__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* tm, int x, int r0, int r1, int r2, int r3,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
      "%4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
      "l"(tm), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------------------
// launcher of the token-block FFN on tcgen05 (pi_tc.cu)

// true if the shape takes the tcgen05 token-block path
bool tc_ffn_supported(int wtype, int ptype, int d, int B);
// workspace bytes of that path: split-K dots, fp16 activation rows, partial outputs
size_t tc_ws_bytes(int d, int ffn, int B);
// y[B, d] = b2 + sum over the list [0, n_hot) ++ idx[0, *count) of act(...) W_downT[j]
cudaError_t launch_tc_ffn(int act, const void* h, int B, int d, int ffn, int n_hot, const int32_t* idx,
                          const int32_t* count, const void* wg, const void* wu, const void* wd, const float* b1,
                          const float* b2, float* y, void* scratch, Ctrl* ctrl, int sms, cudaStream_t st);

}  // namespace pi
