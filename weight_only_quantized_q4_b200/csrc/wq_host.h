// wq_host.h — host-side status helpers shared by the libwq translation units.
#pragma once

#include <string>

namespace wq {

// Record a failure message for wq_last_error() on this thread and return code.
int fail(int code, const std::string& msg);
// Clear nothing, return WQ_OK (kept for symmetry at call sites).
int ok();
// Record the liveness label of the kernel the current call launched.
void set_last_kernel(const std::string& label);

}  // namespace wq
