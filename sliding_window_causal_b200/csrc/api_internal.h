// api_internal.h: helpers that the library's translation units share (not exported in
// include/swa.h). The message set here is what swa_last_error() returns.
#pragma once

namespace swa_internal {
// Record `msg` as the calling thread's last error and return `code`.
int set_error(int code, const char* msg);
// Clear the calling thread's last error and return SWA_OK.
int clear_error();
}  // namespace swa_internal
