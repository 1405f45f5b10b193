// Sequence-parallel covariance side of the full-Kalman scan: the covariance at every chunk start from
// composed chunk transfer matrices, so that the chunks' gains can then be computed all at once.
//
// Kalman Delta Networks, Abstract: exact covariance tracking is a dense, state-dependent Riccati
// recursion that does not map onto GPU-parallel scans, while Moebius maps compose.  The dense recursion
// is itself a matrix Moebius (linear-fractional) map of P: with P = X Y^-1, one token is
//   [X; Y] <- M_t [X; Y],  M_t = [[a^2 I, Qn I], [a^2 k k^T / r, I + Qn k k^T / r]]
// (predict P^- = a^2 P + Qn I, then the update P = P^- (I + k k^T P^- / r)^-1), and a chunk of C tokens is
// the product of its tokens' matrices.  That product has a closed form: with alpha_t = prod a^2,
// beta_t = a_t^2 beta_{t-1} + Qn_t, beta_{t,j} the noise accumulated over tokens j+1..t,
//   M_chunk = [[alpha I, beta I], [0, I]] + U W^T,  U[:, j] = [beta_{C,j} k_j; k_j],
//   W = B (diag(r) - Cs^T)^-1,  B[:, t] = [alpha_t k_t; beta_t k_t],  Cs_tj = (k_j . k_t) beta_{t,j} (j < t),
// one C x C triangular solve per chunk.  Three kernels:
//   riccati_chunk_map_kernel  every chunk's W, U coefficients, alpha and beta, all chunks at once;
//   riccati_chain_kernel      [X; Y] from [P0; I] through the chunk maps, one CTA per head and block of 16
//                             columns (the columns of [X; Y] transform independently, and each may be
//                             rescaled freely: P = X Y^-1 does not change), storing [X; Y] at the start of
//                             every run of cps chunks;
//   riccati_extract_kernel    P = X Y^-1 at every run start (LU with partial pivoting of Y^T, then
//                             P^T = Y^-T X^T by substitution, symmetrised), all runs at once.
// The chunked covariance kernel then walks every run from its own start covariance, all runs in parallel.
#include <cuda_runtime.h>

#include "chunk.h"
#include "common.cuh"
#include "kernels.h"

namespace kdn {

namespace {

constexpr int kRC = 64;  // tokens per chunk, as the covariance kernel's chunks

// ---------------------------------------------------------------------------------------- chunk maps
// W [BH][nch][kRC][2D] (row t: column t of W, i.e. the coefficients of the chunk's t-th rank-1 term),
// ucoef [BH][nch][kRC] (beta_{C,j}), ab [BH][nch][2] (alpha, beta of the whole chunk).
template <int D>
__global__ void __launch_bounds__(2 * D) riccati_chunk_map_kernel(RiccatiArgs p) {
  constexpr int NT = 2 * D, C = kRC, LK = D + 1, LC = C + 1;
  extern __shared__ float msm[];
  float (*kf)[LK] = reinterpret_cast<float (*)[LK]>(msm);  // [C][LK] the chunk's keys
  __shared__ float Cs[C][LC];     // (k_j . k_t) beta_{t,j} for j < t
  __shared__ float sa[C], sr[C], sq[C], salpha[C], sbeta[C];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x, c = blockIdx.y, L = p.L, nch = (L + C - 1) / C;
  const int t0 = c * C, n = min(C, L - t0);
  const size_t tok0 = (size_t)bh * L;
  const __nv_bfloat16* kb = reinterpret_cast<const __nv_bfloat16*>(p.k);

  for (int idx = tid; idx < C * D; idx += NT) {
    const int t = idx / D, i = idx % D;
    kf[t][i] = t < n ? __bfloat162float(kb[(tok0 + t0 + t) * D + i]) : 0.f;
  }
  if (tid < C) {
    const bool ok = tid < n;
    const size_t ti = tok0 + t0 + tid;
    sa[tid] = ok ? (p.a != nullptr ? p.a[ti] : 1.f) : 1.f;
    sr[tid] = ok ? p.r[ti] : 1.f;
    sq[tid] = ok ? (p.qn != nullptr ? p.qn[ti] : p.qn_scalar) : 0.f;
  }
  __syncthreads();
  if (warp == 0 && lane == 0) {  // alpha_t, beta_t (64 steps)
    float al = 1.f, be = 0.f;
    for (int t = 0; t < C; ++t) {
      const float a2 = sa[t] * sa[t];
      al *= a2;
      be = fmaf(a2, be, sq[t]);
      salpha[t] = al, sbeta[t] = be;
    }
  }
  // K K^T into Cs (full), then the noise factors
  for (int idx = tid; idx < C * C; idx += NT) {
    const int t = idx / C, j = idx % C;
    float acc = 0.f;
    if (j < t) {
#pragma unroll 8
      for (int i = 0; i < D; ++i) acc = fmaf(kf[t][i], kf[j][i], acc);
    }
    Cs[t][j] = acc;
  }
  __syncthreads();
  float* ucoef = p.map_u + ((size_t)bh * nch + c) * C;
  if (tid < C) {  // beta_{t,j} down column j (t > j), folded into Cs; beta_{C,j} is the U coefficient
    const int j = tid;
    float acc = 0.f;
    for (int t = j + 1; t < C; ++t) {
      acc = fmaf(sa[t] * sa[t], acc, sq[t]);
      Cs[t][j] *= acc;
    }
    ucoef[j] = acc;
  }
  __syncthreads();
  if (tid == 0) {
    float* ab = p.map_ab + ((size_t)bh * nch + c) * 2;
    ab[0] = salpha[C - 1], ab[1] = sbeta[C - 1];
  }
  // row rho of W: w_t = (b_t + sum_{j<t} Cs_tj w_j) / r_t, b_t = (alpha_t or beta_t) k_t[rho mod D]
  {
    const int rho = tid, i = rho % D;
    const float* sc = rho < D ? salpha : sbeta;
    float w[C];
#pragma unroll
    for (int t = 0; t < C; ++t) {
      float acc = sc[t] * kf[t][i];
#pragma unroll
      for (int j = 0; j < t; ++j) acc = fmaf(Cs[t][j], w[j], acc);
      w[t] = acc / sr[t];
    }
    float* Wc = p.map_w + ((size_t)bh * nch + c) * C * NT;
#pragma unroll
    for (int t = 0; t < C; ++t) Wc[(size_t)t * NT + rho] = w[t];
  }
}

// ---------------------------------------------------------------------------------------- the chain
// [X; Y] (2D x 16 columns of this CTA) from [P0; I] through the chunk maps; xy [BH][runs][2D][D] gets the pair
// entering every run (every cps-th chunk).  Each chunk's W^T (64 KB at d = 128), keys and U coefficients are
// copied asynchronously, the next chunk's while the current one is applied.
constexpr int kRCols = 16, kChainThreads = 512;

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

template <int D>
struct ChainLayout {
  static constexpr int C = kRC, R2 = 2 * D, NC = kRCols;
  static constexpr int WS = R2 + 4;  // padded row stride of W^T: rows t, t+1 start 4 banks apart
  static constexpr int W_FLOATS = C * WS, K_HALVES = C * D;
  // floats: 2 W^T buffers, 2 U buffers, [X; Y], Z, column scales; then 2 bf16 key buffers
  static constexpr int OFF_U = 2 * W_FLOATS, OFF_XY = OFF_U + 2 * C, OFF_Z = OFF_XY + R2 * NC, OFF_S = OFF_Z + C * NC;
  static constexpr int OFF_K = OFF_S + NC;  // in floats, 16-byte aligned below
  static constexpr size_t BYTES = (size_t)OFF_K * 4 + 2 * (size_t)K_HALVES * 2;
  static_assert(OFF_K % 4 == 0, "key buffers must start 16-byte aligned");
};

template <int D>
__global__ void __launch_bounds__(kChainThreads, 1) riccati_chain_kernel(RiccatiArgs p) {
  using Ly = ChainLayout<D>;
  constexpr int NT = kChainThreads, C = kRC, R2 = 2 * D, NC = kRCols, WS = Ly::WS;
  constexpr int PER_Z = C * NC / NT, PER_X = D * NC / NT;
  extern __shared__ __align__(16) float rsm[];
  float* XY = rsm + Ly::OFF_XY;  // [R2][NC]
  float* Z = rsm + Ly::OFF_Z;    // [C][NC]
  float* scl = rsm + Ly::OFF_S;  // [NC] column maxima, then scales
  __nv_bfloat16* kbuf = reinterpret_cast<__nv_bfloat16*>(rsm + Ly::OFF_K);
  const int tid = threadIdx.x;
  const int bh = blockIdx.x, col0 = blockIdx.y * NC, L = p.L, nch = (L + C - 1) / C;
  const int cps = p.cps, runs = (nch + cps - 1) / cps;
  const __nv_bfloat16* kg = reinterpret_cast<const __nv_bfloat16*>(p.k) + (size_t)bh * L * D;
  // chunk c's W^T, U coefficients and keys into buffer c & 1 (chunks before the last run start are full)
  auto fetch = [&](int c) {
    const int b = c & 1;
    float* Wd = rsm + b * Ly::W_FLOATS;
    const float* Wc = p.map_w + ((size_t)bh * nch + c) * C * R2;
    for (int idx = tid; idx < C * R2 / 4; idx += NT) {
      const int t = idx / (R2 / 4), q = idx % (R2 / 4);
      cp_async16(Wd + t * WS + 4 * q, Wc + (size_t)t * R2 + 4 * q);
    }
    if (tid < C / 4) cp_async16(rsm + Ly::OFF_U + b * C + 4 * tid, p.map_u + ((size_t)bh * nch + c) * C + 4 * tid);
    const __nv_bfloat16* kc = kg + (size_t)c * C * D;
    for (int idx = tid; idx < C * D / 8; idx += NT) cp_async16(kbuf + b * Ly::K_HALVES + 8 * idx, kc + 8 * idx);
    cp_async_commit();
  };

  for (int idx = tid; idx < R2 * NC; idx += NT) {
    const int rho = idx / NC, cc = idx % NC, col = col0 + cc;
    XY[idx] = rho < D ? p.P0[((size_t)bh * D + rho) * D + col] : (rho - D == col ? 1.f : 0.f);
  }
  const int last = (runs - 1) * cps;  // the maps of the chunks past the last run start are not needed
  if (last > 0) fetch(0);
  for (int c = 0; c <= last; ++c) {
    __syncthreads();
    if (c % cps == 0) {
      float* xyc = p.xy + ((size_t)bh * runs + c / cps) * R2 * D;
      for (int idx = tid; idx < R2 * NC; idx += NT) xyc[(size_t)(idx / NC) * D + col0 + idx % NC] = XY[idx];
    }
    if (c == last) break;
    if (c + 1 < last) fetch(c + 1);
    else cp_async_commit();  // an empty group keeps the wait count uniform
    const float* ab = p.map_ab + ((size_t)bh * nch + c) * 2;
    const float alpha = __ldg(ab), beta = __ldg(ab + 1);
    const float* Ws = rsm + (c & 1) * Ly::W_FLOATS;
    const float* uc = rsm + Ly::OFF_U + (c & 1) * C;
    const __nv_bfloat16* kf = kbuf + (c & 1) * Ly::K_HALVES;
    cp_async_wait_one();  // this chunk's copies have landed (the next chunk's may still be in flight)
    __syncthreads();
    // Z = W^T [X; Y]
#pragma unroll
    for (int u = 0; u < PER_Z; ++u) {
      const int idx = tid + NT * u, t = idx / NC, cc = idx % NC;
      float acc = 0.f;
#pragma unroll 8
      for (int rho = 0; rho < R2; rho += 4) {
        const float4 w = *reinterpret_cast<const float4*>(Ws + t * WS + rho);
        acc = fmaf(w.x, XY[rho * NC + cc], acc);
        acc = fmaf(w.y, XY[(rho + 1) * NC + cc], acc);
        acc = fmaf(w.z, XY[(rho + 2) * NC + cc], acc);
        acc = fmaf(w.w, XY[(rho + 3) * NC + cc], acc);
      }
      Z[idx] = acc;
    }
    __syncthreads();
    // [X; Y] <- [alpha X + beta Y; Y] + U Z, U[:, t] = [u_t k_t; k_t]
    float nx[PER_X], ny[PER_X];
#pragma unroll
    for (int u = 0; u < PER_X; ++u) {
      const int idx = tid + NT * u, i = idx / NC, cc = idx % NC;
      float sx = 0.f, sy = 0.f;
#pragma unroll 8
      for (int t = 0; t < C; ++t) {
        const float kz = __bfloat162float(kf[t * D + i]) * Z[t * NC + cc];
        sx = fmaf(uc[t], kz, sx);
        sy += kz;
      }
      const float x = XY[i * NC + cc], y = XY[(D + i) * NC + cc];
      nx[u] = fmaf(alpha, x, fmaf(beta, y, sx));
      ny[u] = y + sy;
    }
    if (tid < NC) scl[tid] = 0.f;
    __syncthreads();
#pragma unroll
    for (int u = 0; u < PER_X; ++u) {
      const int idx = tid + NT * u, i = idx / NC, cc = idx % NC;
      XY[i * NC + cc] = nx[u], XY[(D + i) * NC + cc] = ny[u];
      atomicMax(reinterpret_cast<int*>(&scl[cc]), __float_as_int(fabsf(ny[u])));  // non-negative floats order as ints
    }
    __syncthreads();
    // rescale each column of [X; Y] by a power of two near 1 / max |Y column| (exact; P = X Y^-1 unchanged)
    for (int idx = tid; idx < R2 * NC; idx += NT) {
      const int e = (__float_as_int(scl[idx % NC]) >> 23) & 0xff;
      XY[idx] *= __int_as_float((254 - min(max(e, 1), 253)) << 23);
    }
  }
}

// ---------------------------------------------------------------------------------------- P = X Y^-1
// At every run start: LU with partial pivoting of Y^T (one warp picks each pivot, swaps and forms the
// multipliers; every thread updates the trailing block), then P^T = Y^-T X^T by forward and back
// substitution over the 128 right-hand sides, symmetrised.
constexpr int kGJThreads = 256;

template <int D>
__global__ void __launch_bounds__(kGJThreads, 1) riccati_extract_kernel(RiccatiArgs p) {
  constexpr int NT = kGJThreads, LD = D + 1;
  extern __shared__ float gsm[];
  float* A = gsm;                   // [D][LD]: Y^T, then its LU factors
  float* Bm = gsm + D * LD;         // [D][LD]: X^T, then P^T
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x, sg = blockIdx.y, runs = gridDim.y;
  const float* xyc = p.xy + ((size_t)bh * runs + sg) * 2 * D * D;
  float* Pc = p.P_starts + ((size_t)bh * runs + sg) * D * D;
  if (sg == 0) {  // the first run starts from [P0; I]: P0 itself
    for (int idx = tid; idx < D * D; idx += NT) Pc[idx] = xyc[idx];
    return;
  }
  for (int idx = tid; idx < D * D; idx += NT) {
    const int rr = idx / D, cc = idx % D;  // X[rr][cc], Y[rr][cc]
    Bm[cc * LD + rr] = xyc[(size_t)rr * D + cc];
    A[cc * LD + rr] = xyc[(size_t)(D + rr) * D + cc];
  }
  __syncthreads();
  bool singular = false;
  // --- LU with partial pivoting: A = P L U (rows of A and Bm swapped together)
  for (int k = 0; k < D; ++k) {
    if (warp == 0) {
      float best = -1.f;
      int bi = k;
      for (int i = k + lane; i < D; i += 32) {
        const float v = fabsf(A[i * LD + k]);
        if (v > best) best = v, bi = i;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ob > best || (ob == best && oi < bi)) best = ob, bi = oi;
      }
      if (bi != k)
        for (int j = lane; j < D; j += 32) {
          float t = A[k * LD + j];
          A[k * LD + j] = A[bi * LD + j], A[bi * LD + j] = t;
          t = Bm[k * LD + j];
          Bm[k * LD + j] = Bm[bi * LD + j], Bm[bi * LD + j] = t;
        }
      __syncwarp();
      const float piv = A[k * LD + k];
      singular |= !(fabsf(piv) > 0.f);
      const float inv = 1.f / piv;
      for (int i = k + 1 + lane; i < D; i += 32) A[i * LD + k] *= inv;  // multipliers l_ik
    }
    __syncthreads();
    // trailing update A[i][j] -= l_ik A[k][j] (i, j > k)
    const int w = D - 1 - k;
    for (int idx = tid; idx < w * w; idx += NT) {
      const int i = k + 1 + idx / w, j = k + 1 + idx % w;
      A[i * LD + j] = fmaf(-A[i * LD + k], A[k * LD + j], A[i * LD + j]);
    }
    __syncthreads();
  }
  // --- forward substitution L Z = Bm (unit lower), then back substitution U P^T = Z; 128 columns in parallel
  for (int k = 0; k < D - 1; ++k) {
    for (int idx = tid; idx < (D - 1 - k) * D; idx += NT) {
      const int i = k + 1 + idx / D, j = idx % D;
      Bm[i * LD + j] = fmaf(-A[i * LD + k], Bm[k * LD + j], Bm[i * LD + j]);
    }
    __syncthreads();
  }
  for (int k = D - 1; k >= 0; --k) {
    const float inv = 1.f / A[k * LD + k];
    for (int j = tid; j < D; j += NT) Bm[k * LD + j] *= inv;
    __syncthreads();
    for (int idx = tid; idx < k * D; idx += NT) {
      const int i = idx / D, j = idx % D;
      Bm[i * LD + j] = fmaf(-A[i * LD + k], Bm[k * LD + j], Bm[i * LD + j]);
    }
    __syncthreads();
  }
  if (singular && tid == 0) raise_status(p.status, kStatusNumeric);
  // Bm = P^T; write P symmetrised
  for (int idx = tid; idx < D * D; idx += NT) {
    const int rr = idx / D, cc = idx % D;
    Pc[idx] = 0.5f * (Bm[cc * LD + rr] + Bm[rr * LD + cc]);
  }
}

template <int D>
cudaError_t launch_riccati_typed(const RiccatiArgs& a, cudaStream_t st) {
  const int nch = (a.L + kRC - 1) / kRC, runs = (nch + a.cps - 1) / a.cps, last = (runs - 1) * a.cps;
  cudaError_t e;
  if (last > 0) {  // the maps of the chunks before the last run start
    const size_t map_smem = (size_t)kRC * (D + 1) * 4;
    e = cudaFuncSetAttribute(riccati_chunk_map_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)map_smem);
    if (e != cudaSuccess) return e;
    riccati_chunk_map_kernel<D><<<dim3(a.BH, last), 2 * D, map_smem, st>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const size_t chain_smem = ChainLayout<D>::BYTES;
  e = cudaFuncSetAttribute(riccati_chain_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)chain_smem);
  if (e != cudaSuccess) return e;
  riccati_chain_kernel<D><<<dim3(a.BH, D / kRCols), kChainThreads, chain_smem, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t lu_smem = (size_t)2 * D * (D + 1) * 4;
  e = cudaFuncSetAttribute(riccati_extract_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lu_smem);
  if (e != cudaSuccess) return e;
  riccati_extract_kernel<D><<<dim3(a.BH, runs), kGJThreads, lu_smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

size_t riccati_scratch_bytes(int d, int BH, int L, int cps) {
  auto r256 = [](size_t n) { return (n + 255) / 256 * 256; };
  if (cps < 1) return 0;
  const size_t nch = ((size_t)L + kRC - 1) / kRC, chunks = (size_t)BH * nch;
  const size_t runs = (size_t)BH * ((nch + cps - 1) / cps);
  return r256(chunks * kRC * 2 * d * 4) + r256(chunks * kRC * 4) + r256(chunks * 2 * 4) + r256(runs * 2 * d * d * 4) +
         r256(runs * d * d * 4);
}

cudaError_t launch_riccati_starts(int d, const RiccatiArgs& args, cudaStream_t stream) {
  if (args.BH <= 0 || args.L <= 0) return cudaSuccess;
  if (args.cps < 1) return cudaErrorInvalidValue;
  if (d == 64) return launch_riccati_typed<64>(args, stream);
  if (d == 128) return launch_riccati_typed<128>(args, stream);
  return cudaErrorInvalidValue;
}

}  // namespace kdn
