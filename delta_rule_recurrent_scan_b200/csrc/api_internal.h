// Host-side helpers shared by the C-ABI entry points (validation, errors, dispatch).
#pragma once

#include <cuda_runtime.h>

#include <string>

#include "../../include/kdn.h"
#include "device_guard.h"

namespace kdn {
namespace api {

constexpr size_t kStatusBytes = 256;  // leading status word of every workspace

struct CudaDeviceOps {
  static int get(int* dev) { return static_cast<int>(cudaGetDevice(dev)); }
  static int set(int dev) { return static_cast<int>(cudaSetDevice(dev)); }
};
// Declared first in every entry point that launches: restores the caller's device on return.
using DeviceGuard = ScopedDevice<CudaDeviceOps>;

kdn_status fail(kdn_status s, const std::string& msg);
kdn_status ok();
kdn_status check_dims(const kdn_dims* d);
kdn_status check_ptr(const void* p, const char* name, size_t align, bool allow_null);
// Make the device that owns ``p`` current for the rest of the guard's scope.
kdn_status use_device_of(const void* p, DeviceGuard& guard);
kdn_status cuda_status(cudaError_t e, const char* what);
// Segments per head for a request (1 = the serial scan); an explicit request that cannot be served fails.
kdn_status resolve_segments(kdn_variant var, const kdn_dims* d, int* P_out);
// Device address, on the current device, of the no-alloc entry point's static scratch (its first 256
// bytes are that entry point's status word).
kdn_status noalloc_scratch_on_current_device(void** out);

// Full or diagonal Kalman scan with an explicit workspace (status word + gain scratch).
kdn_status kalman_scan(kdn_variant var, const kdn_dims* dims, const void* q, const void* k, const void* v,
                       const float* a, const float* r, const float* qn, float qn_scalar, float* S, float* P,
                       void* o, float* m, void* workspace, size_t workspace_bytes, void* stream);

}  // namespace api
}  // namespace kdn
