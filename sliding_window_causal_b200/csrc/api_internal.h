// api_internal.h: helpers that the library's translation units share (not exported in
// include/swa.h). The message set here is what swa_last_error() returns.
#pragma once

#include <stdint.h>

namespace swa_internal {
// Record `msg` as the calling thread's last error and return `code`.
int set_error(int code, const char* msg);
// Clear the calling thread's last error and return SWA_OK.
int clear_error();
// Every check swa_forward_ex makes that needs no device (sizes, dtype, scale, null
// pointers, strides, alignment, launch-size limits), in its order. Returns SWA_OK or the
// refusal with its message set; on SWA_OK with B*H*T > 0, st holds the effective element
// strides q, k, v, out x (b, h, t). Nothing touches the device.
int check_forward(const char* fn, const void* q, const void* k, const void* v, const void* out, int64_t B,
                  int64_t H, int64_t T, int64_t D, int64_t W, double scale, const int64_t* strides, int dtype,
                  int64_t st[4][3]);
}  // namespace swa_internal
