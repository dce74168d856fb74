// abi_internal.h - helpers shared by the two host-side files of the C ABI
// (fp8attn_abi.cu: device-buffer entries; fp8attn_host.cu: the host-buffer
// pipeline).  Not part of the public interface.
#pragma once
#include <cstdint>
#include <string>

#include "fp8attn.h"

namespace fp8attn {

// Record `why` as this host thread's last error and return `status`.
int fail(int status, const std::string& why);
void clear_error();
const char* last_error();

// Every argument check of the attention entry points, before any driver call.
// host_buffers: Q, K, V, O are host memory (no alignment rule; no row range).
// Returns a negative status (last error set), 0 (valid), or 1 (valid, B*H*N = 0).
int validate(const fp8attn_params* p, bool host_buffers);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace fp8attn
