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

}  // namespace pi
