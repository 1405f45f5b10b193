// Chunked tensor-core scan kernels (sm_100a).
#include "chunk.h"

namespace kdn {

bool chunk_supported(kdn_variant, const kdn_dims&) { return false; }

void chunk_plan(kdn_variant, const kdn_dims&, int* launches, const char** kernel, const char** arith) {
  *launches = 0, *kernel = "", *arith = "";
}

cudaError_t launch_chunk(kdn_variant, const kdn_dims&, const ChunkArgs&, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace kdn
