// Surprise-cache read (A Hippocampus for Linear Attention, sections 3.3-3.4, Eq. (6)-(7)).
//
// Each head keeps the exact (k, v) of the w tokens with the largest surprise m_t seen so far.  Token t of
// block b reads with a softmax, temperature 1, over the cache of blocks 0..b-1, the causal tokens of its
// own block and one null sink (a logit, no value):
//
//   o_t = sum_{j in V_t} softmax_j(q~_t^T k~_j / sqrt(d_k)) v_j,   q~ = RMSNorm_gq(q), k~ = RMSNorm_gk(k),
//   RMSNorm_g(x) = x / sqrt(mean(x^2) + 1e-6) * g.
//
// One CTA of 256 threads per head walks the blocks in order.  Per block: normalise the block's q and k
// into shared memory, score the 64 queries against the (at most) 64 cache keys and 64 block keys with
// 4 x 8 register tiles, softmax each row with the sink, multiply by the values the same way, write o, and
// merge the block into the cache: every candidate's rank is the number of candidates with a larger m
// (ties towards the earlier token), and the w best move to the front.  fp32 throughout.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace kdn {

namespace {

constexpr int kHThreads = 256;
constexpr int kHMax = 64;     // block and cache capacity
constexpr int kHCols = 2 * kHMax;

template <int DK, int DV>
struct HolaLayout {
  static constexpr int LDK = DK + 4, LDV = DV + 4, LDP = kHCols + 4;
  static constexpr int LDT = (DK > DV ? DK : DV) + 4;   // scratch rows: queries, then the cache merge
  static constexpr int OFF_K = 0;                       // [128][LDK] keys: rows 0..63 cache, 64..127 block
  static constexpr int OFF_V = OFF_K + kHCols * LDK;    // [128][LDV] values
  static constexpr int OFF_Q = OFF_V + kHCols * LDV;    // [64][LDT] normalised queries / merge scratch
  static constexpr int OFF_P = OFF_Q + kHMax * LDT;     // [64][LDP] logits, then probabilities / scratch
  static constexpr int FLOATS = OFF_P + kHMax * (LDP > LDT ? LDP : LDT);
  static constexpr int SMEM = FLOATS * 4;
};

__device__ __forceinline__ float load_x(const void* base, size_t i, int dtype) {
  return dtype == kBF16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i])
                        : reinterpret_cast<const float*>(base)[i];
}

// Candidate c precedes d in the cache order: larger m first, then the earlier token.
__device__ __forceinline__ bool before(float mc, int ic, float md, int id) { return mc > md || (mc == md && ic < id); }

template <int DK, int DV>
__global__ void __launch_bounds__(kHThreads) hola_read_kernel(HolaArgs p) {
  using Lay = HolaLayout<DK, DV>;
  extern __shared__ float hs[];
  float* Ks = hs + Lay::OFF_K;
  float* Vs = hs + Lay::OFF_V;
  float* Qs = hs + Lay::OFF_Q;
  float* Ps = hs + Lay::OFF_P;
  __shared__ float mc[kHCols];      // m of the cache (0..63) and of the block (64..127); -inf = empty
  __shared__ int ic[kHCols];        // their token indices
  __shared__ int newpos[kHCols];    // position in the merged cache, or -1
  __shared__ int ncache;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x, h = bh % p.H;
  const int L = p.L, blk = p.block, w = p.w;
  const size_t tok0 = (size_t)bh * L;
  const float scale = rsqrtf((float)DK);
  const float sink = p.sink[h];
  if (tid < kHCols) mc[tid] = -INFINITY, ic[tid] = -1;
  if (tid == 0) ncache = 0;
  // empty cache rows are multiplied by probability 0: they must hold finite numbers
  for (int e = tid; e < kHMax * Lay::LDK; e += kHThreads) Ks[e] = 0.f;
  for (int e = tid; e < kHMax * Lay::LDV; e += kHThreads) Vs[e] = 0.f;
  __syncthreads();

  for (int b0 = 0; b0 < L; b0 += blk) {
    const int nb = min(blk, L - b0);
    // ---- the block's normalised queries and keys, values, surprise (one warp per token)
    for (int i = warp; i < kHMax; i += kHThreads / 32) {
      const bool valid = i < nb;
      const size_t t = tok0 + b0 + i;
      float qss = 0.f, kss = 0.f;
      float qv[(DK + 31) / 32], kv[(DK + 31) / 32];
#pragma unroll
      for (int u = 0; u < (DK + 31) / 32; ++u) {
        const int d = lane + 32 * u;
        qv[u] = (valid && d < DK) ? load_x(p.q, t * DK + d, p.in_dtype) : 0.f;
        kv[u] = (valid && d < DK) ? load_x(p.k, t * DK + d, p.in_dtype) : 0.f;
        qss = fmaf(qv[u], qv[u], qss), kss = fmaf(kv[u], kv[u], kss);
      }
      qss = warp_sum(qss), kss = warp_sum(kss);
      const float qr = rsqrtf(qss / DK + 1e-6f), kr = rsqrtf(kss / DK + 1e-6f);
#pragma unroll
      for (int u = 0; u < (DK + 31) / 32; ++u) {
        const int d = lane + 32 * u;
        if (d < DK) {
          Qs[i * Lay::LDT + d] = qv[u] * qr * p.gamma_q[d];
          Ks[(kHMax + i) * Lay::LDK + d] = valid ? kv[u] * kr * p.gamma_k[d] : 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < (DV + 31) / 32; ++u) {
        const int d = lane + 32 * u;
        if (d < DV) Vs[(kHMax + i) * Lay::LDV + d] = valid ? load_x(p.v, t * DV + d, p.in_dtype) : 0.f;
      }
      if (lane == 0) {
        mc[kHMax + i] = valid ? p.m[t] : -INFINITY;
        ic[kHMax + i] = valid ? b0 + i : -1;
      }
    }
    __syncthreads();

    // ---- logits: 64 queries x 128 keys, 4 x 8 tiles (rows 4 rt.., columns 8 ct..)
    const int rt = tid >> 4, ct = tid & 15;
    {
      float acc[4][8];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[r][c] = 0.f;
#pragma unroll 4
      for (int d = 0; d < DK; d += 4) {
        float4 qa[4], kb[8];
#pragma unroll
        for (int r = 0; r < 4; ++r) qa[r] = *reinterpret_cast<const float4*>(Qs + (4 * rt + r) * Lay::LDT + d);
#pragma unroll
        for (int c = 0; c < 8; ++c) kb[c] = *reinterpret_cast<const float4*>(Ks + (ct + 16 * c) * Lay::LDK + d);
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            acc[r][c] = fmaf(qa[r].x, kb[c].x, acc[r][c]);
            acc[r][c] = fmaf(qa[r].y, kb[c].y, acc[r][c]);
            acc[r][c] = fmaf(qa[r].z, kb[c].z, acc[r][c]);
            acc[r][c] = fmaf(qa[r].w, kb[c].w, acc[r][c]);
          }
      }
      const int nc = ncache;
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int i = 4 * rt + r, j = ct + 16 * c;
          const bool vis = j < kHMax ? j < nc : (j - kHMax <= i && j - kHMax < nb);
          Ps[i * Lay::LDP + j] = vis ? acc[r][c] * scale : -INFINITY;
        }
    }
    __syncthreads();

    // ---- softmax of each row with the sink (four threads per row, 32 columns each)
    {
      const int i = tid >> 2, part = tid & 3;
      float* row = Ps + i * Lay::LDP + 32 * part;
      float mx = sink;
#pragma unroll 8
      for (int j = 0; j < 32; ++j) mx = fmaxf(mx, row[j]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      float sum = 0.f;
#pragma unroll 8
      for (int j = 0; j < 32; ++j) {
        const float e = __expf(row[j] - mx);
        row[j] = e;
        sum += e;
      }
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      const float inv = 1.f / (sum + __expf(sink - mx));
#pragma unroll 8
      for (int j = 0; j < 32; ++j) row[j] *= inv;
    }
    __syncthreads();

    // ---- o = P V: 64 x DV, tiles of 4 rows x (DV / 16) columns
    {
      constexpr int CV = DV / 16 > 0 ? DV / 16 : 1;  // columns per thread
      float acc[4][CV];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < CV; ++c) acc[r][c] = 0.f;
      if (ct * CV < DV) {
#pragma unroll 4
        for (int j = 0; j < kHCols; ++j) {
          float pr[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) pr[r] = Ps[(4 * rt + r) * Lay::LDP + j];
#pragma unroll
          for (int c = 0; c < CV; ++c) {
            const float vv = Vs[j * Lay::LDV + ct + 16 * c];
#pragma unroll
            for (int r = 0; r < 4; ++r) acc[r][c] = fmaf(pr[r], vv, acc[r][c]);
          }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int i = 4 * rt + r;
          if (i < nb) {
#pragma unroll
            for (int c = 0; c < CV; ++c)
              if (ct + 16 * c < DV) p.o[(tok0 + b0 + i) * DV + ct + 16 * c] = acc[r][c];
          }
        }
      }
    }
    __syncthreads();

    // ---- merge the block into the cache: rank of every candidate, the best w kept, moved to the front
    if (tid < kHCols) {
      const float m0 = mc[tid];
      const int i0 = ic[tid];
      int rank = 0;
      for (int c = 0; c < kHCols; ++c) rank += (c != tid && ic[c] >= 0 && before(mc[c], ic[c], m0, i0)) ? 1 : 0;
      newpos[tid] = (i0 >= 0 && rank < w) ? rank : -1;
    }
    __syncthreads();
    // copy the kept rows into the scratch buffers (keys into Ps, values into Qs), then back to rows 0..
    for (int e = tid; e < kHCols * DK; e += kHThreads) {
      const int c = e / DK, d = e % DK;
      const int np = newpos[c];
      if (np >= 0) Ps[np * Lay::LDP + d] = Ks[c * Lay::LDK + d];
    }
    for (int e = tid; e < kHCols * DV; e += kHThreads) {
      const int c = e / DV, d = e % DV;
      const int np = newpos[c];
      if (np >= 0) Qs[np * Lay::LDT + d] = Vs[c * Lay::LDV + d];
    }
    float m_keep = -INFINITY;
    int i_keep = -1;
    if (tid < kHCols && newpos[tid] >= 0) m_keep = mc[tid], i_keep = ic[tid];
    __syncthreads();
    if (tid < kHCols) mc[tid] = -INFINITY, ic[tid] = -1;
    __syncthreads();
    if (i_keep >= 0) {
      mc[newpos[tid]] = m_keep;
      ic[newpos[tid]] = i_keep;
    }
    for (int e = tid; e < kHMax * DK; e += kHThreads) {
      const int c = e / DK, d = e % DK;
      Ks[c * Lay::LDK + d] = Ps[c * Lay::LDP + d];
    }
    for (int e = tid; e < kHMax * DV; e += kHThreads) {
      const int c = e / DV, d = e % DV;
      Vs[c * Lay::LDV + d] = Qs[c * Lay::LDT + d];
    }
    __syncthreads();
    if (tid == 0) {
      int n = 0;
      for (int c = 0; c < kHMax; ++c) n += ic[c] >= 0 ? 1 : 0;
      ncache = n;
    }
    __syncthreads();
  }

  // ---- the final cache's token indices, ascending (-1 = empty)
  if (p.cache != nullptr && tid < w) {
    const int mine = tid < kHMax ? ic[tid] : -1;
    int pos = -1;
    if (mine >= 0) {
      pos = 0;
      for (int c = 0; c < kHMax; ++c) pos += (ic[c] >= 0 && ic[c] < mine) ? 1 : 0;
    }
    if (mine >= 0) p.cache[(size_t)bh * w + pos] = mine;
    const int n = ncache;
    if (tid >= n) p.cache[(size_t)bh * w + tid] = -1;
  }
}

template <int DK, int DV>
cudaError_t launch_typed(const HolaArgs& p, int BH, cudaStream_t stream) {
  using Lay = HolaLayout<DK, DV>;
  cudaError_t e = cudaFuncSetAttribute(hola_read_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::SMEM);
  if (e != cudaSuccess) return e;
  hola_read_kernel<DK, DV><<<BH, kHThreads, Lay::SMEM, stream>>>(p);
  return cudaGetLastError();
}

template <int DK>
cudaError_t launch_dv(int dv, const HolaArgs& p, int BH, cudaStream_t stream) {
  switch (dv) {
    case 16: return launch_typed<DK, 16>(p, BH, stream);
    case 32: return launch_typed<DK, 32>(p, BH, stream);
    case 64: return launch_typed<DK, 64>(p, BH, stream);
    case 128: return launch_typed<DK, 128>(p, BH, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_hola_read(int dk, int dv, const HolaArgs& p, int BH, cudaStream_t stream) {
  if (hola_tc_supported(dk, dv, p.in_dtype, p.block)) return launch_hola_read_tc(p, BH, stream);
  switch (dk) {
    case 16: return launch_dv<16>(dv, p, BH, stream);
    case 32: return launch_dv<32>(dv, p, BH, stream);
    case 64: return launch_dv<64>(dv, p, BH, stream);
    case 128: return launch_dv<128>(dv, p, BH, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kdn
