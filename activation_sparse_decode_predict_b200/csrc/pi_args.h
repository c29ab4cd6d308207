// pi_args.h -- host-side argument checks shared by the entry points of libpi
// (defined in pi_api.cu).  Each returns PI_OK, or the error status after
// setting the text pi_last_error() returns; none touches the device.
#pragma once
#include <stddef.h>
#include <stdint.h>

#include "pi.h"

namespace pi {

// Text returned by pi_last_error() in this thread.
void set_last_error(const char* msg);
// Descriptor fields and token-block size (the rules every entry point shares).
pi_status check_desc(const pi_ffn_desc* d, int32_t batch);
// Non-NULL and `align`-byte aligned; `name` goes into the error text.
pi_status check_ptr(const void* p, size_t align, const char* name);

// Token-block element type of a descriptor: fp32 with fp32 predictors, fp16
// with fp16 or Q4_0 predictors.
inline int token_type(const pi_ffn_desc* d) { return d->ptype == PI_F32 ? PI_F32 : PI_F16; }

// Scales of a Q4_0 predictor matrix [rows, cols]: they follow its codes
// (rows x cols/2 bytes) in the same buffer.  NULL for other predictor types.
inline const void* pred_scales(const pi_ffn_desc* d, const void* P, int64_t rows, int64_t cols) {
  if (d->ptype != PI_Q4_0 || !P) return nullptr;
  return static_cast<const uint8_t*>(P) + rows * (cols / 2);
}

}  // namespace pi
