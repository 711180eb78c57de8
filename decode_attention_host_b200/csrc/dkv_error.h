// dkv_error.h -- the library-wide "last error" slot behind dkv_last_error_string().
#pragma once
#include <string>

namespace dkv {
// Records msg as the calling thread's last error and returns code.
int set_error(int code, const std::string& msg);
}  // namespace dkv
