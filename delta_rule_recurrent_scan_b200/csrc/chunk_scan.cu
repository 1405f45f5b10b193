// Host side of the chunked scans: tensor maps of the bf16 inputs, the support check and the dispatch to
// the warp-specialised tensor-core kernel (chunk_scan_ws.cu, d_k = d_v = 64 or 128) and, for full Kalman
// with one segment per head, the chunked covariance side before it (pside.cu).
#include <cuda.h>

#include <mutex>

#include "chunk.h"
#include "common.cuh"
#include "kernels.h"

namespace kdn {

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [BH][L][d] bf16 viewed as a 3-D tensor; 64 x 64 boxes with the 128-byte swizzle.
bool make_tmap_impl(CUtensorMap* tm, const void* base, int BH, int L, int d) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)L, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)L * d * 2};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool make_bf16_tmap(CUtensorMap* tm, const void* base, int BH, int L, int d) { return make_tmap_impl(tm, base, BH, L, d); }

bool chunk_supported(kdn_variant variant, const kdn_dims& d) {
  (void)variant;
  return d.in_dtype == KDN_BF16 && d.dk == d.dv && (d.dk == 64 || d.dk == 128) && (d.chunk == 0 || d.chunk == 64) &&
         d.L > 0 && encode_fn() != nullptr;
}

void chunk_plan(kdn_variant variant, const kdn_dims& d, int* launches, const char** kernel, const char** arith) {
  *launches = variant == KDN_KALMAN_FULL ? 2 : 1;
  *kernel = variant == KDN_KALMAN_FULL ? "kalman_pside_kernel" : "chunk_scan_ws_kernel";
  *arith = "bf16-tc";
}

cudaError_t launch_chunk(kdn_variant variant, const kdn_dims& d, const ChunkArgs& a, cudaStream_t stream) {
  if (variant == KDN_KALMAN_FULL) {
    // covariance side first (chunked Woodbury / LDL): per-token gains into the workspace, then the S side
    float* gains = reinterpret_cast<float*>(a.workspace);
    cudaError_t e = launch_kalman_pside(d.dk, a.k, a.a, a.r, a.qn, a.qn_scalar, a.P, gains, a.status, a.BH, a.L, stream);
    if (e != cudaSuccess) return e;
    return launch_chunk_sside(variant, d, a, gains, stream);
  }
  return launch_chunk_sside(variant, d, a, nullptr, stream);
}

cudaError_t launch_chunk_sside(kdn_variant variant, const kdn_dims& d, const ChunkArgs& a, const float* gains,
                               cudaStream_t stream) {
  return launch_chunk_ws(variant, d, a, gains, stream);
}

}  // namespace kdn
