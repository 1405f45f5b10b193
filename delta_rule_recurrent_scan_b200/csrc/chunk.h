// Internal interface of the chunked (tensor-core) scan kernels.
#pragma once

#include <cuda_runtime.h>

#include "../../include/kdn.h"

namespace kdn {

struct ChunkArgs {
  const void* q;
  const void* k;
  const void* v;
  const float* beta;  // delta
  const float* a;     // or nullptr
  const float* r;     // Kalman
  const float* qn;    // Kalman, or nullptr
  float qn_scalar;
  float* S;
  float* P;           // full: [BH, dk, dk]; diagonal: p [BH, dk]
  void* o;
  float* m;
  int out_dtype;
  int BH;
  int L;
  unsigned* status;
  void* workspace;    // past the status word
};

// True when the chunked tensor-core kernel serves this request.
bool chunk_supported(kdn_variant variant, const kdn_dims& dims);
void chunk_plan(kdn_variant variant, const kdn_dims& dims, int* launches, const char** kernel, const char** arith);
cudaError_t launch_chunk(kdn_variant variant, const kdn_dims& dims, const ChunkArgs& args, cudaStream_t stream);

}  // namespace kdn
