// Sequence-parallel covariance side of the full-Kalman scan: the covariance at the start of every run of
// chunks from chained chunk transfer matrices, so that the runs' gains can then be computed all at once.
//
// Kalman Delta Networks, Abstract: exact covariance tracking is a dense, state-dependent Riccati
// recursion that does not map onto GPU-parallel scans, while Moebius maps compose.  The dense recursion
// is itself a matrix Moebius (linear-fractional) map of P: with P = X Y^-1, one token is
//   [X; Y] <- M_t [X; Y],  M_t = [[a^2 I, Qn I], [a^2 k k^T / r, I + Qn k k^T / r]]
// (predict P^- = a^2 P + Qn I, then the update P = P^- (I + k k^T P^- / r)^-1), and a chunk of C tokens is
// the product of its tokens' matrices.  That product has a closed form: with alpha_t = prod a^2,
// beta_t = a_t^2 beta_{t-1} + Qn_t, beta_{t,j} the noise accumulated over tokens j+1..t,
//   M_chunk = [[alpha I, beta I], [0, I]] + U W^T,  U[:, j] = [beta_{C,j} k_j; k_j],
//   W = B G,  G = (diag(r) - Cs^T)^-1,  B[:, t] = [alpha_t k_t; beta_t k_t],  Cs_tj = (k_j . k_t) beta_{t,j} (j < t).
// Applied to [X; Y] without forming W: Z = G^T (diag(alpha_t) K X + diag(beta_t) K Y), then
// X' = alpha_C X + beta_C Y + K^T diag(beta_{C,j}) Z and Y' = Y + K^T Z.  Three kernels:
//   riccati_chunk_map_kernel  every chunk's G, U coefficients and per-token alpha, beta, all chunks at
//                             once; G^T = (diag(r) - Cs)^-1 = diag(1/r) (I - Cs diag(1/r))^-1, a unit lower
//                             triangular inverse;
//   riccati_chain_kernel      [X; Y] from [P0; I] through the chunk maps, one CTA per head and block of 8
//                             columns (the columns of [X; Y] transform independently, and each may be
//                             rescaled freely: P = X Y^-1 does not change), storing [X; Y] at the start of
//                             every run of cps chunks;
//   riccati_extract_kernel    P = X Y^-1 at every run start: Gauss-Jordan with partial pivoting on
//                             [Y^T | X^T] held in registers, then symmetrised, all runs at once.
// The chunked covariance kernel then walks every run from its own start covariance, all runs in parallel.
#include <cuda_runtime.h>

#include "chunk.h"
#include "chunk_common.cuh"
#include "common.cuh"
#include "kernels.h"

namespace kdn {

namespace {

constexpr int kRC = 64;  // tokens per chunk, as the covariance kernel's chunks
constexpr int kMapThreads = 256;

// Eight bf16 values (one 16-byte load) to floats.
__device__ __forceinline__ void bf16x8_to_f32(const uint4 raw, float* out) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(h[e]);
    out[2 * e] = f.x, out[2 * e + 1] = f.y;
  }
}

// ---------------------------------------------------------------------------------------- chunk maps
// map_g [BH][nch][C][C]: G^T (row t = column t of G), map_u [BH][nch][C]: beta_{C,j},
// map_ab [BH][nch][C][2]: alpha_t, beta_t.  Only chunks before the last run start are mapped (all full).
template <int D>
__global__ void __launch_bounds__(kMapThreads) riccati_chunk_map_kernel(RiccatiArgs p) {
  constexpr int NT = kMapThreads, C = kRC, LK = D + 4, LC = chunk::kLD;
  static_assert(C == chunk::kC && LK >= LC, "the key buffer is reused for the inverse");
  extern __shared__ __align__(16) float msm[];
  float* kf = msm;          // [C][LK] keys, later T = (I - Cs diag(1/r))^-1 with row stride LC
  float* Cs = kf + C * LK;  // [C][LC]: (k_j . k_t) beta_{t,j} for j < t, then -Cs_tj / r_j
  __shared__ float sa[C], sr[C], sq[C];
  const int tid = threadIdx.x;
  const int bh = blockIdx.x, c = blockIdx.y, nch = (p.L + C - 1) / C;
  const size_t tok0 = (size_t)bh * p.L + (size_t)c * C;
  const __nv_bfloat16* kg = reinterpret_cast<const __nv_bfloat16*>(p.k) + tok0 * D;
  const size_t map = (size_t)bh * nch + c;

  for (int idx = tid; idx < C * D / 8; idx += NT) {
    const int t = idx / (D / 8), i8 = idx % (D / 8);
    float f[8];
    bf16x8_to_f32(*reinterpret_cast<const uint4*>(kg + (size_t)t * D + 8 * i8), f);
    *reinterpret_cast<float4*>(kf + t * LK + 8 * i8) = make_float4(f[0], f[1], f[2], f[3]);
    *reinterpret_cast<float4*>(kf + t * LK + 8 * i8 + 4) = make_float4(f[4], f[5], f[6], f[7]);
  }
  if (tid < C) {
    const size_t ti = tok0 + tid;
    sa[tid] = p.a != nullptr ? p.a[ti] : 1.f;
    sr[tid] = p.r[ti];
    sq[tid] = p.qn != nullptr ? p.qn[ti] : p.qn_scalar;
  }
  __syncthreads();
  {  // K K^T: thread (tb, jb) takes rows tb + 16u and jb + 16w (eight consecutive rows per quarter warp)
    const int tb = tid / 16, jb = tid % 16;
    float acc[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < 4; ++w) acc[u][w] = 0.f;
#pragma unroll 2
    for (int i = 0; i < D; i += 4) {
      float4 kt[4], kj[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) kt[u] = *reinterpret_cast<const float4*>(kf + (tb + 16 * u) * LK + i);
#pragma unroll
      for (int w = 0; w < 4; ++w) kj[w] = *reinterpret_cast<const float4*>(kf + (jb + 16 * w) * LK + i);
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          float x = acc[u][w];
          x = fmaf(kt[u].x, kj[w].x, x);
          x = fmaf(kt[u].y, kj[w].y, x);
          x = fmaf(kt[u].z, kj[w].z, x);
          acc[u][w] = fmaf(kt[u].w, kj[w].w, x);
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int t = tb + 16 * u, j = jb + 16 * w;
        Cs[t * LC + j] = j < t ? acc[u][w] : 0.f;
      }
  }
  __syncthreads();
  if (tid < C) {  // beta_{t,j} down column j (t > j) and 1 / r_j folded into Cs; beta_{C,j} is the U coefficient
    const int j = tid;
    const float nir = -1.f / sr[j];
    float acc = 0.f;
    for (int t = j + 1; t < C; ++t) {
      acc = fmaf(sa[t] * sa[t], acc, sq[t]);
      Cs[t * LC + j] *= acc * nir;
    }
    p.map_u[map * C + j] = acc;
  } else if (tid == C) {  // alpha_t, beta_t
    float al = 1.f, be = 0.f;
    float* ab = p.map_ab + map * 2 * C;
    for (int t = 0; t < C; ++t) {
      const float a2 = sa[t] * sa[t];
      al *= a2;
      be = fmaf(a2, be, sq[t]);
      ab[2 * t] = al, ab[2 * t + 1] = be;
    }
  }
  __syncthreads();
  // T = (I + N)^-1 with N = -Cs diag(1/r) strictly lower; G^T = diag(1/r) T
  chunk::invert_unit_lower_64(Cs, kf, tid, [] { __syncthreads(); });
  float* Gt = p.map_g + map * C * C;
  for (int idx = tid; idx < C * C; idx += NT) {
    const int t = idx / C, sx = idx % C;
    Gt[idx] = sx <= t ? kf[t * LC + sx] / sr[t] : 0.f;
  }
}

// ---------------------------------------------------------------------------------------- the chain
// [X; Y] (2D x 8 columns of this CTA, held transposed) from [P0; I] through the chunk maps; xy [BH][runs][2D][D]
// gets the pair entering every run (every cps-th chunk).  The next chunk's keys, G^T and coefficients are
// copied asynchronously while the current chunk is applied.  A chunk, with 256 threads in register blocks:
//   R = diag(alpha_t) K X + diag(beta_t) K Y   thread: 2 tokens x 2 columns over half of i (pairs summed by shuffle)
//   Z = G^T R                                   thread: 1 token x 2 columns
//   X' = alpha_C X + beta_C Y + K^T diag(u) Z,  thread: d/64 rows x 2 columns
//   Y' = Y + K^T Z
// Each column of [X; Y] is rescaled by a power of two (exact; X Y^-1 does not change) from the maximum of
// |Y| over the column one chunk earlier, which needs no extra pass or barrier.
constexpr int kRCols = 8, kChainThreads = 256;

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

template <int D>
struct ChainLayout {
  static constexpr int C = kRC, NC = kRCols;
  static constexpr int LG = C + 4;   // row strides in floats (bf16 for keys), chosen so that the rows a warp
  static constexpr int LX = D + 4;   // reads together start 4 banks apart
  static constexpr int LRS = NC + 4;  // R row stride: eight consecutive rows start on distinct bank quads
  static constexpr int LKB = D + 8;
  static constexpr int OFF_G = 0;                    // 2 x [C][LG]  G^T
  static constexpr int OFF_AB = OFF_G + 2 * C * LG;  // 2 x [C][2]   alpha_t, beta_t
  static constexpr int OFF_U = OFF_AB + 2 * 2 * C;   // 2 x [C]      beta_{C,j}
  static constexpr int OFF_X = OFF_U + 2 * C;        // [NC][LX]     X^T
  static constexpr int OFF_Y = OFF_X + NC * LX;      // [NC][LX]     Y^T
  static constexpr int OFF_R = OFF_Y + NC * LX;      // [C][LRS]     R
  static constexpr int OFF_Z = OFF_R + C * LRS;      // [C][NC]      Z
  static constexpr int OFF_ZU = OFF_Z + C * NC;      // [C][NC]      diag(u) Z
  static constexpr int OFF_S = OFF_ZU + C * NC;      // 2 x [NC]     column maxima of |Y| (by chunk parity)
  static constexpr int OFF_K = OFF_S + 2 * NC;       // 2 x [C][LKB] bf16 keys
  static constexpr int K_HALVES = C * LKB;
  static constexpr size_t BYTES = (size_t)OFF_K * 4 + 2 * (size_t)K_HALVES * 2;
  static_assert(OFF_AB % 4 == 0 && OFF_U % 4 == 0 && OFF_X % 4 == 0 && OFF_Y % 4 == 0 && OFF_R % 4 == 0 &&
                    OFF_K % 4 == 0,
                "16-byte aligned regions");
};

template <int D>
__global__ void __launch_bounds__(kChainThreads, 2) riccati_chain_kernel(RiccatiArgs p) {
  using Ly = ChainLayout<D>;
  constexpr int NT = kChainThreads, C = kRC, NC = kRCols, LG = Ly::LG, LX = Ly::LX, LRS = Ly::LRS, LKB = Ly::LKB;
  extern __shared__ __align__(16) float rsm[];
  float* Xt = rsm + Ly::OFF_X;
  float* Yt = rsm + Ly::OFF_Y;
  float* Rs = rsm + Ly::OFF_R;
  float* Zs = rsm + Ly::OFF_Z;
  float* Zu = rsm + Ly::OFF_ZU;
  float* scl = rsm + Ly::OFF_S;
  __nv_bfloat16* kbuf = reinterpret_cast<__nv_bfloat16*>(rsm + Ly::OFF_K);
  const int tid = threadIdx.x;
  const int bh = blockIdx.x, col0 = blockIdx.y * NC, nch = (p.L + C - 1) / C;
  const int cps = p.cps, runs = (nch + cps - 1) / cps;
  const __nv_bfloat16* kg = reinterpret_cast<const __nv_bfloat16*>(p.k) + (size_t)bh * p.L * D;
  // chunk c's G^T, alpha/beta, U coefficients and keys into buffer c & 1 (chunks before the last run are full)
  auto fetch = [&](int c) {
    const int b = c & 1;
    const size_t map = (size_t)bh * nch + c;
    const float* gsrc = p.map_g + map * C * C;
    for (int idx = tid; idx < C * C / 4; idx += NT) {
      const int t = idx / (C / 4), q = idx % (C / 4);
      cp_async16(rsm + Ly::OFF_G + b * C * LG + t * LG + 4 * q, gsrc + t * C + 4 * q);
    }
    if (tid < 2 * C / 4) cp_async16(rsm + Ly::OFF_AB + b * 2 * C + 4 * tid, p.map_ab + map * 2 * C + 4 * tid);
    else if (tid < 2 * C / 4 + C / 4) {
      const int q = tid - 2 * C / 4;
      cp_async16(rsm + Ly::OFF_U + b * C + 4 * q, p.map_u + map * C + 4 * q);
    }
    const __nv_bfloat16* kc = kg + (size_t)c * C * D;
    for (int idx = tid; idx < C * D / 8; idx += NT) {
      const int t = idx / (D / 8), q = idx % (D / 8);
      cp_async16(kbuf + b * Ly::K_HALVES + t * LKB + 8 * q, kc + (size_t)t * D + 8 * q);
    }
    cp_async_commit();
  };

  for (int idx = tid; idx < NC * D; idx += NT) {
    const int cc = idx / D, i = idx % D;
    Xt[cc * LX + i] = p.P0[((size_t)bh * D + i) * D + col0 + cc];
    Yt[cc * LX + i] = i == col0 + cc ? 1.f : 0.f;
  }
  if (tid < NC) scl[NC + tid] = 1.f;  // the scale chunk 0 applies: 1
  const int last = (runs - 1) * cps;  // the chunks past the last run start are not needed
  if (last > 0) fetch(0);
  for (int c = 0; c <= last; ++c) {
    __syncthreads();
    if (c % cps == 0) {
      float* xyc = p.xy + ((size_t)bh * runs + c / cps) * 2 * D * D;
      for (int idx = tid; idx < 2 * D * NC; idx += NT) {
        const int rho = idx / NC, cc = idx % NC;
        xyc[(size_t)rho * D + col0 + cc] = rho < D ? Xt[cc * LX + rho] : Yt[cc * LX + rho - D];
      }
    }
    if (c == last) break;
    if (c + 1 < last) fetch(c + 1);
    else cp_async_commit();  // an empty group keeps the wait count uniform
    const float* Gt = rsm + Ly::OFF_G + (c & 1) * C * LG;
    const float* ab = rsm + Ly::OFF_AB + (c & 1) * 2 * C;
    const float* uc = rsm + Ly::OFF_U + (c & 1) * C;
    const __nv_bfloat16* kf = kbuf + (c & 1) * Ly::K_HALVES;
    cp_async_wait_one();  // this chunk's copies have landed (the next chunk's may still be in flight)
    __syncthreads();
    // ---- R = diag(alpha) K X + diag(beta) K Y: thread (token quad tq, column pair cp, i part ip of 4); the
    // parts hold interleaved i pairs and are summed by shuffles (ip = lane bits 0..1)
    {
      const int ip = tid & 3, cp = (tid >> 2) & 3, tq = tid >> 4;
      const int t0 = 4 * tq, c0 = 2 * cp;
      float kx[4][2], ky[4][2];
#pragma unroll
      for (int u = 0; u < 4; ++u) kx[u][0] = kx[u][1] = ky[u][0] = ky[u][1] = 0.f;
#pragma unroll 4
      for (int i = 2 * ip; i < D; i += 8) {
        float2 kv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          kv[u] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(kf + (t0 + u) * LKB + i));
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const float2 x = *reinterpret_cast<const float2*>(Xt + (c0 + w) * LX + i);
          const float2 y = *reinterpret_cast<const float2*>(Yt + (c0 + w) * LX + i);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            kx[u][w] = fmaf(kv[u].x, x.x, fmaf(kv[u].y, x.y, kx[u][w]));
            ky[u][w] = fmaf(kv[u].x, y.x, fmaf(kv[u].y, y.y, ky[u][w]));
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          kx[u][w] += __shfl_xor_sync(0xffffffffu, kx[u][w], 1);
          kx[u][w] += __shfl_xor_sync(0xffffffffu, kx[u][w], 2);
          ky[u][w] += __shfl_xor_sync(0xffffffffu, ky[u][w], 1);
          ky[u][w] += __shfl_xor_sync(0xffffffffu, ky[u][w], 2);
        }
      // lane ip writes token t0 + ip
      float rx0 = kx[0][0], rx1 = kx[0][1], ry0 = ky[0][0], ry1 = ky[0][1];
#pragma unroll
      for (int u = 1; u < 4; ++u)
        if (ip == u) rx0 = kx[u][0], rx1 = kx[u][1], ry0 = ky[u][0], ry1 = ky[u][1];
      const int t = t0 + ip;
      const float al = ab[2 * t], be = ab[2 * t + 1];
      *reinterpret_cast<float2*>(Rs + t * LRS + c0) = make_float2(fmaf(al, rx0, be * ry0), fmaf(al, rx1, be * ry1));
    }
    if (tid < NC) scl[(c & 1) * NC + tid] = 0.f;  // nobody reads this parity's maxima any more
    __syncthreads();
    // ---- Z = G^T R and diag(u) Z: thread (token quad tq, column quad cq, s part sp of 8; sp = lane bits 0..2)
    {
      const int sp = tid & 7, cq = (tid >> 3) & 1, tq = tid >> 4, t0 = 4 * tq, c0 = 4 * cq;
      float z[4][4];
#pragma unroll
      for (int u = 0; u < 4; ++u) z[u][0] = z[u][1] = z[u][2] = z[u][3] = 0.f;
#pragma unroll
      for (int sx = sp; sx < C; sx += 8) {
        const float4 r4 = *reinterpret_cast<const float4*>(Rs + sx * LRS + c0);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float g = Gt[(t0 + u) * LG + sx];
          z[u][0] = fmaf(g, r4.x, z[u][0]);
          z[u][1] = fmaf(g, r4.y, z[u][1]);
          z[u][2] = fmaf(g, r4.z, z[u][2]);
          z[u][3] = fmaf(g, r4.w, z[u][3]);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          z[u][w] += __shfl_xor_sync(0xffffffffu, z[u][w], 1);
          z[u][w] += __shfl_xor_sync(0xffffffffu, z[u][w], 2);
          z[u][w] += __shfl_xor_sync(0xffffffffu, z[u][w], 4);
        }
      if (sp < 4) {  // lane sp writes token t0 + sp
        float4 zz = make_float4(z[0][0], z[0][1], z[0][2], z[0][3]);
#pragma unroll
        for (int u = 1; u < 4; ++u)
          if (sp == u) zz = make_float4(z[u][0], z[u][1], z[u][2], z[u][3]);
        const int t = t0 + sp;
        const float uu = uc[t];
        *reinterpret_cast<float4*>(Zs + t * NC + c0) = zz;
        *reinterpret_cast<float4*>(Zu + t * NC + c0) = make_float4(uu * zz.x, uu * zz.y, uu * zz.z, uu * zz.w);
      }
    }
    __syncthreads();
    // ---- X, Y updates and rescale: thread (row quad iq, column quad cq, token part tp of 4; tp = lane bits
    // 0..1, interleaved tokens), the parts summed by shuffles; lane tp then finishes row i0 + tp
    {
      const int tp = tid & 3, cq = (tid >> 2) & 1, iq = tid >> 3, i0 = 4 * iq, c0 = 4 * cq;
      constexpr int RPT = D / 32;  // row quads per thread: D = 128 -> 1 quad of 4 rows, D = 64 -> rows of 2
      static_assert(D == 128 || D == 64, "head size");
      constexpr int NR = D == 128 ? 4 : 2;  // rows per thread
      const int r0 = D == 128 ? i0 : 2 * iq;
      float sx[NR][4], sy[NR][4];
#pragma unroll
      for (int e = 0; e < NR; ++e)
#pragma unroll
        for (int w = 0; w < 4; ++w) sx[e][w] = sy[e][w] = 0.f;
#pragma unroll 4
      for (int t = tp; t < C; t += 4) {
        float kv[NR];
        if constexpr (NR == 4) {
          const uint2 raw = *reinterpret_cast<const uint2*>(kf + t * LKB + r0);
          const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
          const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
          kv[0] = lo.x, kv[1] = lo.y, kv[2] = hi.x, kv[3] = hi.y;
        } else {
          const float2 k2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(kf + t * LKB + r0));
          kv[0] = k2.x, kv[1] = k2.y;
        }
        const float4 z = *reinterpret_cast<const float4*>(Zs + t * NC + c0);
        const float4 zu = *reinterpret_cast<const float4*>(Zu + t * NC + c0);
        const float zv[4] = {z.x, z.y, z.z, z.w}, zuv[4] = {zu.x, zu.y, zu.z, zu.w};
#pragma unroll
        for (int e = 0; e < NR; ++e)
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            sx[e][w] = fmaf(kv[e], zuv[w], sx[e][w]);
            sy[e][w] = fmaf(kv[e], zv[w], sy[e][w]);
          }
      }
#pragma unroll
      for (int e = 0; e < NR; ++e)
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          sx[e][w] += __shfl_xor_sync(0xffffffffu, sx[e][w], 1);
          sx[e][w] += __shfl_xor_sync(0xffffffffu, sx[e][w], 2);
          sy[e][w] += __shfl_xor_sync(0xffffffffu, sy[e][w], 1);
          sy[e][w] += __shfl_xor_sync(0xffffffffu, sy[e][w], 2);
        }
      const float alC = ab[2 * (C - 1)], beC = ab[2 * (C - 1) + 1];
      const float* sprev = scl + ((c + 1) & 1) * NC;  // maxima of the previous chunk (1 before chunk 0)
      float* snext = scl + (c & 1) * NC;
      // lane tp finishes row r0 + tp (NR == 4) or, for NR == 2, rows r0 + tp for tp < 2
      if (tp < NR) {
        float ax[4], ay[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) ax[w] = sx[0][w], ay[w] = sy[0][w];
#pragma unroll
        for (int e = 1; e < NR; ++e)
          if (tp == e)
#pragma unroll
            for (int w = 0; w < 4; ++w) ax[w] = sx[e][w], ay[w] = sy[e][w];
        const int i = r0 + tp;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int col = c0 + w;
          const int ex = (__float_as_int(sprev[col]) >> 23) & 0xff;
          const float f = __int_as_float((254 - min(max(ex, 1), 253)) << 23);
          const float x = Xt[col * LX + i], y = Yt[col * LX + i];
          const float yn = f * (y + ay[w]);
          Xt[col * LX + i] = f * fmaf(alC, x, fmaf(beC, y, ax[w]));
          Yt[col * LX + i] = yn;
          atomicMax(reinterpret_cast<int*>(&snext[col]), __float_as_int(fabsf(yn)));  // non-negative floats order as ints
        }
      }
      (void)RPT;
    }
  }
}

// ---------------------------------------------------------------------------------------- chain on tcgen05
// d = 128: one CTA per head carries [X^T | Y^T] in tensor memory (lane = column c of [X; Y], fp32 masters
// X^T and Y^T, their fp16 pairs as the A operands) through the chunk maps with four products per chunk:
//   R^T  = X^T (diag(alpha) K)^T + Y^T (diag(beta) K)^T      A = X^T, Y^T (TMEM)   B = alpha_t k_t, beta_t k_t
//   Z^T  = R^T G                                              A = R^T (TMEM)        B = G^T as stored (rows t)
//   X^T <- alpha_C X^T + beta_C Y^T + Z^T diag(u) K           A = Z^T diag(u)       B = K (d_k contiguous)
//   Y^T <- Y^T + Z^T K                                        A = Z^T               B = K
// then every column is rescaled by a power of two (max |Y| of the column in [1, 2); P = X Y^-1 does not
// change) and the fp16 pairs are formed for the next chunk.  The operands of a chunk (K, alpha K, beta K in
// fp16, G^T in fp16) are built by a second warp group one chunk ahead, in two slots.  Every operand is
// rounded to fp16 once (the keys are exact), with fp32 accumulation and fp32 masters; a float64 model of
// those roundings over a 4096-token head stays near 1e-5 of P.
constexpr int kTcThreads = 512;  // 256 chain + 256 preparation

struct TcChainLayout {
  static constexpr int PANEL = 64 * 128;                // 64 rows x 64 fp16
  static constexpr int OFF_K = 0;                       // K: 2 panels
  static constexpr int OFF_KA = OFF_K + 2 * PANEL;      // alpha_t k_t
  static constexpr int OFF_KB = OFF_KA + 2 * PANEL;     // beta_t k_t
  static constexpr int OFF_G = OFF_KB + 2 * PANEL;      // G^T (row t, columns s): 1 panel
  static constexpr int SLOT = OFF_G + PANEL;
  static constexpr int SMEM = 2 * SLOT + 1024;          // + alignment slack
  // tensor memory columns
  static constexpr uint32_t T_XM = 0, T_YM = 128, T_XP = 256, T_YP = 320, T_R = 384, T_Z = 448;
};

__global__ void __launch_bounds__(kTcThreads, 1) riccati_chain_tc_kernel(RiccatiArgs p) {
  constexpr int D = 128, C = kRC;
  using Ly = TcChainLayout;
  extern __shared__ uint8_t tsm_raw[];
  uint8_t* tsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tsm_raw) + 1023) & ~uintptr_t(1023));
  __shared__ float su[2][C], sac[2][2];
  __shared__ float ymax[2][D];
  __shared__ uint64_t prep_done[2], chain_done[2], bar_m;
  __shared__ uint32_t tmem_base;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x, nch = (p.L + C - 1) / C;
  const int cps = p.cps, runs = (nch + cps - 1) / cps, last = (runs - 1) * cps;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) sm100::mbar_init(&prep_done[i], 1), sm100::mbar_init(&chain_done[i], 1);
    sm100::mbar_init(&bar_m, 1);
    sm100::fence_mbar_init();
  }
  if (warp == 0) {
    sm100::tmem_alloc(&tmem_base, 512);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (tid < 256) {
    // =============================================================== chain: lane c, column half h
    const int qw = warp & 3, half = warp >> 2, col = 32 * qw + lane;
    const uint32_t t_lane = static_cast<uint32_t>(32 * qw) << 16;
    const bool leader = tid == 0;
    bool aborted = false;
    uint32_t ph_m = 0;
    auto gwait = [&](uint64_t* b, uint32_t parity) -> bool {
      bool bad = false;
      if (leader) bad = !sm100::mbar_wait_bounded(b, parity, chunk::kWaitCycles);
      bad = chunk::named_sync_or(1, 256, bad);
      if (bad && leader) raise_status(p.status, kStatusTimeout);
      sm100::tc_fence_after();
      return !bad;
    };
    auto sync_tc = [&] {
      sm100::tc_fence_before();
      chunk::named_sync(1, 256);
      sm100::tc_fence_after();
    };
    // fp16 pairs of 64 master columns (elements 64 half ..) of this lane: 32 pair columns at 32 half
    auto emit_pairs = [&](uint32_t pair_col, const float (&x)[32], int v) {
      float hw[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) hw[e] = __uint_as_float(sm100::pack2_f16(x[2 * e], x[2 * e + 1]));
      sm100::tmem_st16(tmem + t_lane + pair_col + 32 * half + 16 * v, hw);
    };
    // masters at a run start: X rows then Y rows of this run's [X; Y] (row-major 2D x D)
    auto store_start = [&](int run) {
      float* xy = p.xy + ((size_t)bh * runs + run) * 2 * D * D;
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          float x[32];
          sm100::tmem_ld32(tmem + t_lane + (m ? Ly::T_YM : Ly::T_XM) + 64 * half + 32 * v, x);
          sm100::tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 32; ++u) xy[((size_t)m * D + 64 * half + 32 * v + u) * D + col] = x[u];
        }
    };
    // [X; Y] = [P0; I]
#pragma unroll 1
    for (int v = 0; v < 2; ++v) {
      float x[32];
#pragma unroll
      for (int u = 0; u < 32; ++u) x[u] = p.P0[((size_t)bh * D + 64 * half + 32 * v + u) * D + col];
      sm100::tmem_st32(tmem + t_lane + Ly::T_XM + 64 * half + 32 * v, x);
      emit_pairs(Ly::T_XP, x, v);
      sm100::tmem_wait_st();  // (the stores' registers are reused below)
#pragma unroll
      for (int u = 0; u < 32; ++u) x[u] = 64 * half + 32 * v + u == col ? 1.f : 0.f;
      sm100::tmem_st32(tmem + t_lane + Ly::T_YM + 64 * half + 32 * v, x);
      emit_pairs(Ly::T_YP, x, v);
      sm100::tmem_wait_st();
    }
    sm100::tmem_wait_st();
    sync_tc();

    for (int c = 0; c < last && !aborted; ++c) {
      const int s = c & 1;
      if (c % cps == 0) store_start(c / cps);
      if (!gwait(&prep_done[s], (c >> 1) & 1)) { aborted = true; break; }
      const uint32_t slot = sm100::smem_u32(tsm + s * Ly::SLOT);
      // ---- R^T
      if (leader) {
        constexpr uint32_t id = sm100::idesc_f16(128, 64, false, false);
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t b = slot + (m ? Ly::OFF_KB : Ly::OFF_KA) + (ks / 4) * Ly::PANEL + (ks % 4) * 32;
            sm100::mma_bf16_ts(tmem + Ly::T_R, tmem + (m ? Ly::T_YP : Ly::T_XP) + 8 * ks,
                               sm100::smem_desc(b, 16, 1024), id, m > 0 || ks > 0);
          }
        sm100::mma_commit(&bar_m);
      }
      // ---- X^T <- alpha_C X^T + beta_C Y^T while R^T runs (it reads only the pairs)
      {
        const float aC = sac[s][0], bC = sac[s][1];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          float x[16], y[16];
          sm100::tmem_ld16(tmem + t_lane + Ly::T_XM + 64 * half + 16 * v, x);
          sm100::tmem_ld16(tmem + t_lane + Ly::T_YM + 64 * half + 16 * v, y);
          sm100::tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 16; ++u) x[u] = fmaf(aC, x[u], bC * y[u]);
          sm100::tmem_st16(tmem + t_lane + Ly::T_XM + 64 * half + 16 * v, x);
          sm100::tmem_wait_st();
        }
        sm100::tmem_wait_st();
      }
      if (!gwait(&bar_m, ph_m)) { aborted = true; break; }
      ph_m ^= 1;
      // ---- R^T to fp16 pairs in place (tokens 32 half .. + 31), then Z^T = R^T G
      {
        float r[32];
        sm100::tmem_ld32(tmem + t_lane + Ly::T_R + 32 * half, r);
        sm100::tmem_wait_ld();
        float hw[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) hw[e] = __uint_as_float(sm100::pack2_f16(r[2 * e], r[2 * e + 1]));
        sm100::tmem_st16(tmem + t_lane + Ly::T_R + 32 * half, hw);
        sm100::tmem_wait_st();
      }
      sync_tc();
      if (leader) {
        constexpr uint32_t id = sm100::idesc_f16(128, 64, false, false);
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks)
          sm100::mma_bf16_ts(tmem + Ly::T_Z, tmem + Ly::T_R + chunk::tok_pair_col(ks),
                             sm100::smem_desc(slot + Ly::OFF_G + ks * 32, 16, 1024), id, ks > 0);
        sm100::mma_commit(&bar_m);
      }
      if (!gwait(&bar_m, ph_m)) { aborted = true; break; }
      ph_m ^= 1;
      // ---- Z^T pairs in place, Z^T diag(u) pairs over the dead R^T; then the master updates
      {
        float z[32];
        sm100::tmem_ld32(tmem + t_lane + Ly::T_Z + 32 * half, z);
        sm100::tmem_wait_ld();
        float hw[16], hu[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int t = 32 * half + 2 * e;
          hw[e] = __uint_as_float(sm100::pack2_f16(z[2 * e], z[2 * e + 1]));
          hu[e] = __uint_as_float(sm100::pack2_f16(z[2 * e] * su[s][t], z[2 * e + 1] * su[s][t + 1]));
        }
        sm100::tmem_st16(tmem + t_lane + Ly::T_Z + 32 * half, hw);
        sm100::tmem_st16(tmem + t_lane + Ly::T_R + 32 * half, hu);
        sm100::tmem_wait_st();
      }
      sync_tc();
      if (leader) {
        constexpr uint32_t id = sm100::idesc_f16(128, 128, false, true);
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
          for (int ks = 0; ks < C / 16; ++ks)
            sm100::mma_bf16_ts(tmem + (m ? Ly::T_YM : Ly::T_XM), tmem + (m ? Ly::T_Z : Ly::T_R) + chunk::tok_pair_col(ks),
                               sm100::smem_desc(slot + Ly::OFF_K + ks * 2048, Ly::PANEL, 1024), id, true);
        sm100::mma_commit(&chain_done[s]);  // the slot's operands are dead once these complete
        sm100::mma_commit(&bar_m);
      }
      if (!gwait(&bar_m, ph_m)) { aborted = true; break; }
      ph_m ^= 1;
      // ---- rescale every column by a power of two, and the pairs of the next chunk
      {
        float mx = 0.f;
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          float y[32];
          sm100::tmem_ld32(tmem + t_lane + Ly::T_YM + 64 * half + 32 * v, y);
          sm100::tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 32; ++u) mx = fmaxf(mx, fabsf(y[u]));
        }
        ymax[half][col] = mx;
        chunk::named_sync(1, 256);
        const float m = fmaxf(ymax[0][col], ymax[1][col]);
        float sc = 1.f;
        if (m > 0.f && isfinite(m)) {
          const int ey = min((__float_as_int(m) >> 23) & 0xff, 253);
          sc = __int_as_float((254 - ey) << 23);  // 2^(127 - ey): max |Y| of the column into [1, 2)
        } else if (half == 0) {
          raise_status(p.status, kStatusNumeric);
        }
#pragma unroll
        for (int mm = 0; mm < 2; ++mm)
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            float x[32];
            const uint32_t mcol = (mm ? Ly::T_YM : Ly::T_XM) + 64 * half + 32 * v;
            sm100::tmem_ld32(tmem + t_lane + mcol, x);
            sm100::tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 32; ++u) x[u] *= sc;
            sm100::tmem_st32(tmem + t_lane + mcol, x);
            emit_pairs(mm ? Ly::T_YP : Ly::T_XP, x, v);
            sm100::tmem_wait_st();
          }
      }
      sync_tc();
    }
    if (!aborted) store_start(runs - 1);
  } else {
    // =============================================================== preparation of chunk c into slot c & 1
    const int pt = tid - 256;
    const bool leader = pt == 0;
    const __nv_bfloat16* kg = reinterpret_cast<const __nv_bfloat16*>(p.k) + (size_t)bh * p.L * D;
    for (int c = 0; c < last; ++c) {
      const int s = c & 1;
      {
        bool bad = false;
        if (leader && c >= 2) bad = !sm100::mbar_wait_bounded(&chain_done[s], ((c >> 1) & 1) ^ 1, chunk::kWaitCycles);
        bad = chunk::named_sync_or(2, 256, bad);
        if (bad) {
          if (leader) raise_status(p.status, kStatusTimeout);
          break;
        }
      }
      uint8_t* sl = tsm + s * Ly::SLOT;
      const size_t map = (size_t)bh * nch + c;
      const float* ab = p.map_ab + map * 2 * C;
      // K, alpha K, beta K: 64 tokens x 16 chunks of 8 keys, four per thread
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        const int item = pt + 256 * rr, t = item >> 4, q = item & 15;
        float f[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(kg + ((size_t)c * C + t) * D + 8 * q), f);
        const float al = ab[2 * t], be = ab[2 * t + 1];
        float fa[8], fb[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) fa[e] = al * f[e], fb[e] = be * f[e];
        const uint32_t off = (q >> 3) * Ly::PANEL + sm100::sw128_chunk(t, q & 7);
        chunk::store8_f16(sl + Ly::OFF_K, off, f);
        chunk::store8_f16(sl + Ly::OFF_KA, off, fa);
        chunk::store8_f16(sl + Ly::OFF_KB, off, fb);
      }
      // G^T rows t: 64 x 8 chunks, two per thread
      const float* gsrc = p.map_g + map * C * C;
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const int item = pt + 256 * rr, t = item >> 3, q = item & 7;
        const float4 g0 = *reinterpret_cast<const float4*>(gsrc + t * C + 8 * q);
        const float4 g1 = *reinterpret_cast<const float4*>(gsrc + t * C + 8 * q + 4);
        const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        chunk::store8_f16(sl + Ly::OFF_G, sm100::sw128_chunk(t, q), g);
      }
      if (pt < C) su[s][pt] = p.map_u[map * C + pt];
      if (pt == C) sac[s][0] = ab[2 * (C - 1)], sac[s][1] = ab[2 * (C - 1) + 1];
      sm100::fence_async_smem();
      chunk::named_sync(2, 256);
      if (leader) sm100::mbar_arrive(&prep_done[s]);
    }
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 0) sm100::tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------------------- P = X Y^-1
// At every run start, Y^T P^T = X^T by Gauss-Jordan elimination with partial pivoting on the augmented
// [Y^T | X^T] (D x 2D), held in registers: warp w owns rows 8w..8w+7, lane l columns CB l..CB l+CB-1.
// Pivot rows are not swapped but recorded; once every column is eliminated, the row that was pivot for
// column k holds row k of P^T in its right half.  P is written symmetrised.
template <int D>
struct ExtractLayout {
  static constexpr int NT = 4 * D, NW = D / 8, CB = D / 16, LP = D + 1;
  static constexpr int OFF_PROW = D * LP;           // 2 x [2D] normalised pivot row
  static constexpr int OFF_PCOL = OFF_PROW + 4 * D;  // 2 x [D]  pivot column (the multipliers)
  static constexpr int OFF_CV = OFF_PCOL + 2 * D;    // 2 x [NW] candidate pivot magnitudes
  static constexpr int OFF_CR = OFF_CV + 2 * NW;     // 2 x [NW] candidate pivot rows (int)
  static constexpr int OFF_INV = OFF_CR + 2 * NW;    // [D] column of each pivot row (int)
  static constexpr size_t BYTES = (size_t)(OFF_INV + D) * 4;
  static_assert(OFF_PROW % 4 == 0, "16-byte aligned pivot row");
};

template <int D>
__global__ void __launch_bounds__(4 * D, 1) riccati_extract_kernel(RiccatiArgs p) {
  using Ly = ExtractLayout<D>;
  constexpr int NT = Ly::NT, NW = Ly::NW, CB = Ly::CB, LP = Ly::LP;
  extern __shared__ __align__(16) float xsm[];
  float* Pt = xsm;  // [D][LP]: P^T
  float* prow = xsm + Ly::OFF_PROW;
  float* pcol = xsm + Ly::OFF_PCOL;
  float* cand_v = xsm + Ly::OFF_CV;
  int* cand_r = reinterpret_cast<int*>(xsm + Ly::OFF_CR);
  int* invp = reinterpret_cast<int*>(xsm + Ly::OFF_INV);
  __shared__ int bad;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x, sg = blockIdx.y, runs = gridDim.y;
  const float* xyc = p.xy + ((size_t)bh * runs + sg) * 2 * D * D;
  float* Pc = p.P_starts + ((size_t)bh * runs + sg) * D * D;
  if (sg == 0) {  // the first run starts from [P0; I]: P0 itself
    for (int idx = tid; idx < D * D; idx += NT) Pc[idx] = xyc[idx];
    return;
  }
  // a[r][c] = [Y^T | X^T][8 warp + r][CB lane + c]; column j < D of the augmented matrix is row j of Y
  float a[8][CB];
#pragma unroll
  for (int c = 0; c < CB; ++c) {
    const int j = CB * lane + c;
    const float* src = xyc + (size_t)(j < D ? D + j : j - D) * D + 8 * warp;
    const float4 lo = *reinterpret_cast<const float4*>(src), hi = *reinterpret_cast<const float4*>(src + 4);
    a[0][c] = lo.x, a[1][c] = lo.y, a[2][c] = lo.z, a[3][c] = lo.w;
    a[4][c] = hi.x, a[5][c] = hi.y, a[6][c] = hi.z, a[7][c] = hi.w;
  }
  if (tid == 0) bad = 0;
  unsigned used = 0;  // rows of this warp already taken as pivots
  for (int kb = 0; kb < D / CB; ++kb) {
#pragma unroll
    for (int cc = 0; cc < CB; ++cc) {
      const int k = kb * CB + cc, buf = k & 1;
      if (lane == kb) {  // this lane holds column k for the warp's rows: local pivot candidate, multipliers
        float best = -1.f;
        int br = 0;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const float v = fabsf(a[r][cc]);
          if (!((used >> r) & 1u) && v > best) best = v, br = r;
        }
        cand_v[buf * NW + warp] = best;
        cand_r[buf * NW + warp] = 8 * warp + br;
        *reinterpret_cast<float4*>(pcol + buf * D + 8 * warp) = make_float4(a[0][cc], a[1][cc], a[2][cc], a[3][cc]);
        *reinterpret_cast<float4*>(pcol + buf * D + 8 * warp + 4) = make_float4(a[4][cc], a[5][cc], a[6][cc], a[7][cc]);
      }
      __syncthreads();
      // the pivot: largest candidate, the lowest row on ties (every warp reduces the candidates itself)
      float best = lane < NW ? cand_v[buf * NW + lane] : -2.f;
      int pr = lane < NW ? cand_r[buf * NW + lane] : 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int orr = __shfl_xor_sync(0xffffffffu, pr, o);
        if (ob > best || (ob == best && orr < pr)) best = ob, pr = orr;
      }
      if (warp == pr / 8) {  // the pivot's warp publishes the normalised pivot row
        const int rp = pr % 8;
        float row[CB];
#pragma unroll
        for (int c = 0; c < CB; ++c) row[c] = a[0][c];
#pragma unroll
        for (int r = 1; r < 8; ++r)
          if (r == rp)
#pragma unroll
            for (int c = 0; c < CB; ++c) row[c] = a[r][c];
        const float piv = pcol[buf * D + pr];
        if (lane == 0 && !(fabsf(piv) > 0.f && isfinite(piv))) bad = 1;
        const float inv = 1.f / piv;
#pragma unroll
        for (int c = 0; c < CB; ++c) prow[buf * 2 * D + CB * lane + c] = row[c] * inv;
        used |= 1u << rp;
      }
      if (tid == 0) invp[pr] = k;
      __syncthreads();
      float pv[CB], mv[8];
#pragma unroll
      for (int c = 0; c < CB; ++c) pv[c] = prow[buf * 2 * D + CB * lane + c];
#pragma unroll
      for (int r = 0; r < 8; ++r) mv[r] = pcol[buf * D + 8 * warp + r];
      if (warp == pr / 8) {  // the pivot row takes the normalised row, the warp's other rows are eliminated
        const int rp = pr % 8;
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
          for (int c = 0; c < CB; ++c) a[r][c] = r == rp ? pv[c] : fmaf(-mv[r], pv[c], a[r][c]);
      } else {
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
          for (int c = 0; c < CB; ++c) a[r][c] = fmaf(-mv[r], pv[c], a[r][c]);
      }
    }
  }
  // right half of pivot row p = row invp[p] of P^T
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int k = invp[8 * warp + r];
#pragma unroll
    for (int c = 0; c < CB; ++c) {
      const int j = CB * lane + c;
      if (j >= D) Pt[k * LP + j - D] = a[r][c];
    }
  }
  __syncthreads();
  if (bad && tid == 0) raise_status(p.status, kStatusNumeric);
  for (int idx = tid; idx < D * D; idx += NT) {
    const int rr = idx / D, cc = idx % D;
    Pc[idx] = 0.5f * (Pt[cc * LP + rr] + Pt[rr * LP + cc]);
  }
}

template <int D>
cudaError_t launch_riccati_typed(const RiccatiArgs& a, cudaStream_t st) {
  const int nch = (a.L + kRC - 1) / kRC, runs = (nch + a.cps - 1) / a.cps, last = (runs - 1) * a.cps;
  cudaError_t e;
  if (last > 0) {  // the maps of the chunks before the last run start
    const size_t map_smem = (size_t)kRC * ((D + 4) + (kRC + 4)) * 4;
    e = cudaFuncSetAttribute(riccati_chunk_map_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)map_smem);
    if (e != cudaSuccess) return e;
    riccati_chunk_map_kernel<D><<<dim3(a.BH, last), kMapThreads, map_smem, st>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if constexpr (D == 128) {  // the chain on the tensor cores, one CTA per head
    e = cudaFuncSetAttribute(riccati_chain_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, TcChainLayout::SMEM);
    if (e != cudaSuccess) return e;
    riccati_chain_tc_kernel<<<a.BH, kTcThreads, TcChainLayout::SMEM, st>>>(a);
  } else {
    const size_t chain_smem = ChainLayout<D>::BYTES;
    e = cudaFuncSetAttribute(riccati_chain_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)chain_smem);
    if (e != cudaSuccess) return e;
    riccati_chain_kernel<D><<<dim3(a.BH, D / kRCols), kChainThreads, chain_smem, st>>>(a);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t x_smem = ExtractLayout<D>::BYTES;
  e = cudaFuncSetAttribute(riccati_extract_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)x_smem);
  if (e != cudaSuccess) return e;
  riccati_extract_kernel<D><<<dim3(a.BH, runs), ExtractLayout<D>::NT, x_smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

size_t riccati_scratch_bytes(int d, int BH, int L, int cps) {
  auto r256 = [](size_t n) { return (n + 255) / 256 * 256; };
  if (cps < 1) return 0;
  const size_t nch = ((size_t)L + kRC - 1) / kRC, chunks = (size_t)BH * nch;
  const size_t runs = (size_t)BH * ((nch + cps - 1) / cps);
  return r256(chunks * kRC * kRC * 4) + r256(chunks * kRC * 4) + r256(chunks * 2 * kRC * 4) +
         r256(runs * 2 * d * d * 4) + r256(runs * d * d * 4);
}

cudaError_t launch_riccati_starts(int d, const RiccatiArgs& args, cudaStream_t stream) {
  if (args.BH <= 0 || args.L <= 0) return cudaSuccess;
  if (args.cps < 1) return cudaErrorInvalidValue;
  if (d == 64) return launch_riccati_typed<64>(args, stream);
  if (d == 128) return launch_riccati_typed<128>(args, stream);
  return cudaErrorInvalidValue;
}

}  // namespace kdn
