// Full-Kalman scan that allocates nothing: its scratch is a static device array.
//
// kdn_scan_kalman_full asks the caller for a workspace (a 256-byte status word
// plus one fp32 gain per token and key coordinate).  Some callers cannot hand
// one over: code that must not call cudaMalloc once it is running (a server
// that reserves all device memory at start-up and hands out fixed pools, a
// plugin whose host framework owns the device allocator, a real-time loop that
// forbids allocation) and that has no spare buffer of the right size.  This
// entry point runs the same kernels with the scratch in the file-scope array
// below instead.
#include <cuda_runtime.h>

#include <string>

#include "../../include/kdn.h"
#include "api_internal.h"

namespace {

// 256-byte status word, then up to 16 MiB of fp32 gains (B*H*L*d_k <= 4,194,304).
constexpr size_t kNoAllocScratchBytes = kdn::api::kStatusBytes + (size_t(16) << 20);

// Every GPU on which this file's module is loaded holds this array until the process exits.  Under
// lazy module loading that happens at the first no-alloc call (or status read) on the device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

}  // namespace

namespace kdn {
namespace api {

// Device address of the array on the current device.  It is looked up on every call (cheap once the
// module is loaded) rather than cached, so that a device reset, which reloads the module at a new
// address, cannot leave a stale pointer behind.  Under lazy module loading (the CUDA 12 default) the
// first lookup on a device is what loads the module and so reserves the array's memory there.
kdn_status noalloc_scratch_on_current_device(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || p == nullptr) {
    cudaGetLastError();
    return fail(KDN_ERR_CUDA, std::string("cudaGetSymbolAddress of the static scratch: ") + cudaGetErrorString(e));
  }
  *out = p;
  return KDN_OK;
}

}  // namespace api
}  // namespace kdn

extern "C" kdn_status kdn_scan_kalman_full_noalloc(const kdn_dims* dims, const void* q, const void* k, const void* v,
                                                   const float* a, const float* r, const float* qn, float qn_scalar,
                                                   float* S, float* P, void* o, float* m, void* stream) {
  using namespace kdn::api;
  kdn_status st = check_dims(dims);
  if (st != KDN_OK) return st;
  // the static array holds the gains of the serial scan: the library's segment choice is turned off
  kdn_dims d = *dims;
  if (d.segments == 0) d.segments = 1;
  dims = &d;
  int nseg = 1;
  st = resolve_segments(KDN_KALMAN_FULL, dims, &nseg);
  if (st != KDN_OK) return st;
  const size_t need = kdn_workspace_bytes(KDN_KALMAN_FULL, dims);
  if (need > kNoAllocScratchBytes)
    return fail(KDN_ERR_UNSUPPORTED,
                "kdn_scan_kalman_full_noalloc: this scan needs " + std::to_string(need) + " bytes of scratch (" +
                    std::to_string(nseg) + (nseg == 1 ? " segment" : " segments") +
                    " per head) but the static array holds " + std::to_string(kNoAllocScratchBytes) +
                    "; with one segment B*H*L*d_k must be <= 4194304; use kdn_scan_kalman_full with a workspace");
  st = check_ptr(S, "S", 16, false);
  if (st != KDN_OK) return st;
  DeviceGuard guard;
  st = use_device_of(S, guard);  // the scratch address is per device: look it up on the state's device
  if (st != KDN_OK) return st;
  void* scratch = nullptr;
  st = noalloc_scratch_on_current_device(&scratch);
  if (st != KDN_OK) return st;
  return kalman_scan(KDN_KALMAN_FULL, dims, q, k, v, a, r, qn, qn_scalar, S, P, o, m, scratch, kNoAllocScratchBytes,
                     stream);
}
