// pi_noalloc.cu -- pi_predict_static: the predictor without a caller workspace.
//
// Some callers cannot hand the library any scratch memory: hosts that pass a
// plugin only its input and output buffers, or serving loops that must not
// call cudaMalloc once they are running (an allocation can synchronise the
// device and stall every stream).  For them this entry point keeps the
// predictor's scratch -- the fp32 vector u and the per-tile masks and counts --
// in one fixed-size array in device memory that the library itself declares.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds it until the process exits.  Host code cannot use the array's
// name as a device address; its address is fetched once per device with
// cudaGetSymbolAddress (with that device current) and then passed to the
// kernels like any other pointer.
#include <cuda_runtime.h>
#include <mutex>
#include <stdint.h>
#include <stdio.h>

#include "pi.h"
#include "pi_args.h"
#include "pi_kernels_v1.cuh"
#include "pi_layout.h"

namespace {

constexpr size_t kStaticScratchBytes = (size_t)1 << 20;  // 1 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

pi_status err(pi_status st, const char* msg) {
  pi::set_last_error(msg);
  return st;
}

// Device address of g_scratch on the current device (looked up once per device).
pi_status scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return err(PI_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return err(PI_ERR_UNSUPPORTED, "device ordinal above 63");
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || !p) return err(PI_ERR_CUDA, cudaGetErrorString(e));
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return PI_OK;
}

}  // namespace

static_assert(kStaticScratchBytes == PI_STATIC_SCRATCH_BYTES, "header and library agree on the scratch size");

extern "C" {

pi_status pi_predict_static(const pi_ffn_desc* desc, int32_t batch, const void* h, const void* P1, const void* P2,
                            const float* bp, float threshold, int32_t* idx, int32_t* count, void* stream) {
  // the same checks, with the same alignments, as pi_predict: nothing is
  // launched unless every one passes
  pi_status s = pi::check_desc(desc, batch);
  if (s != PI_OK) return s;
  const int ffn = desc->ffn, n_hot = desc->n_hot, r = desc->rank;
  const int C = ffn - n_hot;
  if ((s = pi::check_ptr(h, 16, "h")) != PI_OK) return s;
  if ((s = pi::check_ptr(P1, 16, "P1")) != PI_OK) return s;
  if (C > 0 && (s = pi::check_ptr(P2, 16, "P2")) != PI_OK) return s;
  if (bp && (s = pi::check_ptr(bp, 4, "bp")) != PI_OK) return s;
  if (C > 0 && (s = pi::check_ptr(idx, 4, "idx")) != PI_OK) return s;
  if ((s = pi::check_ptr(count, 4, "count")) != PI_OK) return s;
  // scratch: u [batch, rank] fp32, then the tile masks and tile counts
  const int n_tiles = (C + 255) / 256;
  const size_t u_bytes = pi::align256((size_t)batch * r * 4);
  const size_t m_bytes = pi::align256((size_t)(n_tiles > 0 ? n_tiles : 1) * 8 * 4);
  const size_t c_bytes = pi::align256((size_t)(n_tiles > 0 ? n_tiles : 1) * 4);
  if (u_bytes + m_bytes + c_bytes > kStaticScratchBytes)
    return err(PI_ERR_CAPACITY,
               "pi_predict_static: batch x rank x 4 bytes plus the tile masks exceed the 1 MiB static scratch");
  void* base = nullptr;
  s = scratch_address(&base);
  if (s != PI_OK) return s;
  char* b = static_cast<char*>(base);
  float* u = reinterpret_cast<float*>(b);
  uint32_t* tmask = reinterpret_cast<uint32_t*>(b + u_bytes);
  int* tcount = reinterpret_cast<int*>(b + u_bytes + m_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaError_t e =
      pi::launch_pred_u(desc->ptype, P1, pi::pred_scales(desc, P1, r, desc->d), h, batch, desc->d, r, u, sms, st);
  if (e == cudaSuccess)
    e = pi::launch_pred_score(desc->ptype, P2, pi::pred_scales(desc, P2, C, r), bp, u, batch, r, C, threshold, tmask,
                              tcount, st);
  if (e == cudaSuccess) e = pi::launch_compact(tmask, tcount, C, n_hot, idx, count, st);
  if (e != cudaSuccess) return err(PI_ERR_CUDA, cudaGetErrorString(e));
  return PI_OK;
}

}  // extern "C"
