// Host-side helpers shared by the C-ABI entry points (validation, errors, dispatch).
#pragma once

#include <cuda_runtime.h>

#include <string>

#include "../../include/kdn.h"

namespace kdn {
namespace api {

constexpr size_t kStatusBytes = 256;  // leading status word of every workspace

kdn_status fail(kdn_status s, const std::string& msg);
kdn_status ok();
kdn_status check_dims(const kdn_dims* d);
kdn_status check_ptr(const void* p, const char* name, size_t align, bool allow_null);
kdn_status use_device_of(const void* p);
kdn_status cuda_status(cudaError_t e, const char* what);

// Full or diagonal Kalman scan with an explicit workspace (status word + gain scratch).
kdn_status kalman_scan(kdn_variant var, const kdn_dims* dims, const void* q, const void* k, const void* v,
                       const float* a, const float* r, const float* qn, float qn_scalar, float* S, float* P,
                       void* o, float* m, void* workspace, size_t workspace_bytes, void* stream);

}  // namespace api
}  // namespace kdn
