// Internal interface of the chunked (tensor-core) scan kernels.
#pragma once

#include <cuda.h>
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
  int state_cols;     // columns of a state row: 0 = d_v; 2 d_v = 128 runs the d = 64 chunk kernel on [S | M]
  void* o;            // or nullptr (no read-out)
  float* m;
  int out_dtype;
  int BH;
  int L;
  unsigned* status;
  void* workspace;    // past the status word
};

// [BH][L][d] bf16 viewed as a 3-D tensor map with 64 x 64 boxes and the 128-byte swizzle.
bool make_bf16_tmap(CUtensorMap* tm, const void* base, int BH, int L, int d);

// Covariance side of the full-Kalman scan, chunked (Woodbury / LDL): per-token gains into ``gains``
// ([BH, L, d] fp32) and P updated in place.  d in {64, 128}, bf16 keys.
// P_starts (optional): [BH, ceil(nchunks / cps), d, d], the covariance entering every run of cps chunks;
// every run then walks its chunks in its own CTA (grid BH x runs) and the one holding the last chunk writes P_L.
cudaError_t launch_kalman_pside(int d, const void* k, const float* a, const float* r, const float* qn,
                                float qn_scalar, float* P, float* gains, unsigned* status, int BH, int L,
                                cudaStream_t stream, const float* P_starts = nullptr, int cps = 0);

// Warp-specialised chunk kernel for d_k = d_v = 64 or 128 (preparation of chunk c + 1 beside the state
// chain of chunk c).  ``gains``: full-Kalman per-token gains [BH, L, d] fp32, else unused.  At d = 64,
// args.state_cols = 128 carries a [d, 2 d] state [S | M]: the extra columns see zero values (the map's
// linear part), and o may be nullptr.
cudaError_t launch_chunk_ws(kdn_variant variant, const kdn_dims& dims, const ChunkArgs& args, const float* gains,
                            cudaStream_t stream);

// True when the chunked tensor-core kernel serves this request.
bool chunk_supported(kdn_variant variant, const kdn_dims& dims);
void chunk_plan(kdn_variant variant, const kdn_dims& dims, int* launches, const char** kernel, const char** arith);
cudaError_t launch_chunk(kdn_variant variant, const kdn_dims& dims, const ChunkArgs& args, cudaStream_t stream);
// The memory (S) side alone; full Kalman reads its per-token gains from ``gains`` ([BH, L, dk] fp32).
cudaError_t launch_chunk_sside(kdn_variant variant, const kdn_dims& dims, const ChunkArgs& args, const float* gains,
                               cudaStream_t stream);

}  // namespace kdn
