// Backward of the full-covariance Kalman scan's covariance side (Kalman Delta Networks, Abstract: the dense
// Riccati recursion of the memory's uncertainty; the layers are trained end to end), around the memory
// backward that takes the per-token gains as inputs and writes their gradient dG.
//
// Forward, per token (the symmetric form the forward kernels and the oracle take):
//   P^- = a^2 P + Qn I,  u = P^- k,  s = k^T u + r,  g = u / s,  P <- P^- - u u^T / s.
// Backward, for dg = dG_t: instead of the covariance adjoint Pb the kernels carry its symmetric sum
// M = Pb + Pb^T, which is all the recursion needs while P is symmetric:
//   ds = (-(dg . u) + u^T M u / 2) / s^2,   du = (dg - M u) / s + ds k,
//   dk += ds u + P^- du,   dr = ds,   dQn = tr(M) / 2 + du . k,   da += 2 a (<M, P> / 2 + du . P k),
//   M <- a^2 (M + du k^T + k du^T)            (dP0 = M_0 / 2, the gradient for a symmetric P0).
// One CTA of 4 d threads per head, in row groups of G = 4 R threads: thread g of group n holds rows
// n R .. n R + R - 1 of P (and of M) at the d / G columns 4 G m + 4 g + e (e < 4); R = 2 from d = 32 on (1 at
// d = 16), so that each broadcast vector is read as d / (4 G) float4 per thread, G adjacent float4 per group
// (free of bank conflicts), and a matrix-vector product ends in a reduction over the group's lanes.  Both
// kernels go through the tokens in blocks of kFB, each block's inputs staged in shared memory before it is
// walked (the forward loads the next block into registers while it walks the current one), so no global
// load sits on a token's serial path.  The forward keeps P at every block start; the backward recomputes
// each block's P before every token (to global scratch, in the threads' own float4 order; u and s stay in
// shared memory), then walks the block in reverse with that P streamed back through a two-slot cp.async
// buffer, each thread copying and reading only its own slots.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace kdn {

namespace {

constexpr int kFB = 32;  // tokens per block: inputs staged per block, P checkpointed and recomputed per block

template <int D>
struct FullBwdShape {
  // R rows of P per thread (two from d = 32 on, so that a broadcast vector is read half as often), G = 4 R
  // threads per row group, CW columns per row and thread
  static constexpr int NT = 4 * D, NW = NT / 32, R = D >= 32 ? 2 : 1, G = 4 * R, CW = D / G, NM = CW / 4;
  static constexpr int NV = R * CW / 4;     // float4 per thread per matrix
  static constexpr int KPT = kFB * D / NT;  // block elements per thread when a [kFB, D] block is staged
};

// Thread tid's slot m of a d x d matrix held in thread order: float4 m * NT + tid.
template <int D>
__device__ __forceinline__ float4* slot(float* base, int m, int tid) {
  return reinterpret_cast<float4*>(base) + (size_t)m * FullBwdShape<D>::NT + tid;
}

// Column of register j of thread g of its row group, and that thread's float4 m of a d-vector in shared
// memory: the G threads of a group read G adjacent float4, free of bank conflicts.
template <int G>
__device__ __forceinline__ int colof(int g, int j) { return 4 * G * (j >> 2) + 4 * g + (j & 3); }
template <int G>
__device__ __forceinline__ float4 vec4(const float* v, int m, int g) {
  return reinterpret_cast<const float4*>(v)[G * m + g];
}

// Sum of the NW warp partials v[0 .. NW) (16-byte aligned; NW = 2, 4, 8 or 16), in a short tree.
template <int NW>
__device__ __forceinline__ float sum_parts(const float* v) {
  if constexpr (NW < 4) {
    return v[0] + v[1];
  } else {
    float4 acc = reinterpret_cast<const float4*>(v)[0];
#pragma unroll
    for (int w = 1; w < NW / 4; ++w) {
      const float4 x = reinterpret_cast<const float4*>(v)[w];
      acc.x += x.x, acc.y += x.y, acc.z += x.z, acc.w += x.w;
    }
    return (acc.x + acc.y) + (acc.z + acc.w);
  }
}

// Sum over the G lanes of a row group.
template <int G>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
  for (int o = 1; o < G; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// One forward token of P held by the calling thread (rows r0 .. r0 + R - 1): P <- P^- - u u^T / s.  kv holds the
// token's key (fp32), us receives u (it is also this token's broadcast slot), part the warp partial sums.
// Returns u of the thread's rows and s; one __syncthreads.
template <int D>
__device__ __forceinline__ void cov_step(float (&Pr)[D / 4], const float* kv, float* us, float* part, float at,
                                         float rt, float qt, int tid, unsigned* status,
                                         float (&ui)[FullBwdShape<D>::R], float& s) {
  using Sh = FullBwdShape<D>;
  constexpr int R = Sh::R, G = Sh::G, CW = Sh::CW;
  const int g = tid % G, r0 = (tid / G) * R, lane = tid & 31, warp = tid >> 5;
  const float a2 = at * at;
  float d4[R][4];  // four partial sums per row keep the dependent chains short
#pragma unroll
  for (int r = 0; r < R; ++r) d4[r][0] = d4[r][1] = d4[r][2] = d4[r][3] = 0.f;
#pragma unroll
  for (int m = 0; m < Sh::NM; ++m) {
    const float4 k4 = vec4<G>(kv, m, g);
    const float kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 4 * m + e, x = r * CW + j;
        Pr[x] = fmaf(a2, Pr[x], colof<G>(g, j) == r0 + r ? qt : 0.f);
        d4[r][e] = fmaf(Pr[x], kk[e], d4[r][e]);
      }
  }
  float ku = 0.f;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    ui[r] = group_sum<G>((d4[r][0] + d4[r][1]) + (d4[r][2] + d4[r][3]));
    if (g == 0) ku = fmaf(kv[r0 + r], ui[r], ku);
  }
#pragma unroll
  for (int o = G; o < 32; o <<= 1) ku += __shfl_xor_sync(0xffffffffu, ku, o);
  if (lane == 0) part[warp] = ku;
  if (g == 0)
#pragma unroll
    for (int r = 0; r < R; ++r) us[r0 + r] = ui[r];
  __syncthreads();
  s = rt + sum_parts<Sh::NW>(part);
  if (tid == 0 && status != nullptr && !(s > 0.f && isfinite(s))) raise_status(status, kStatusNumeric);
  float f[R];
#pragma unroll
  for (int r = 0; r < R; ++r) f[r] = ui[r] / s;
#pragma unroll
  for (int m = 0; m < Sh::NM; ++m) {
    const float4 u4 = vec4<G>(us, m, g);
    const float uu[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int e = 0; e < 4; ++e) Pr[r * CW + 4 * m + e] = fmaf(-f[r], uu[e], Pr[r * CW + 4 * m + e]);
  }
}

// The keys of block [t0, t0 + kFB) (zero past L) as fp32 values in registers: element e = tid + NT r is key
// row e / D, coordinate e % D.  Issued a block ahead, stored to shared memory when the block is needed.
template <int D>
__device__ __forceinline__ void load_keys(const FullBwdArgs& p, size_t tok0, int t0, int tid,
                                          float (&kr)[FullBwdShape<D>::KPT]) {
  using Sh = FullBwdShape<D>;
#pragma unroll
  for (int r = 0; r < Sh::KPT; ++r) {
    const int e = tid + Sh::NT * r, t = t0 + e / D;
    kr[r] = t < p.L ? load_elem(p.k, (tok0 + t) * D + e % D, p.in_dtype) : 0.f;
  }
}

template <int D>
__global__ void __launch_bounds__(4 * D, 1) full_cov_forward_kernel(FullBwdArgs p) {
  using Sh = FullBwdShape<D>;
  __shared__ __align__(16) float kf[2][kFB][D];
  __shared__ float sa[2][kFB], sr[2][kFB], sq[2][kFB];
  __shared__ __align__(16) float us[2][D], part[2][Sh::NW];
  constexpr int R = Sh::R, G = Sh::G, CW = Sh::CW;
  const int tid = threadIdx.x, bh = blockIdx.x, L = p.L;
  const int g = tid % G, r0 = (tid / G) * R;
  const size_t tok0 = (size_t)bh * L;
  const int nblk = (L + kFB - 1) / kFB;
  float Pr[R * CW];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int j = 0; j < CW; ++j) {
      const int row = r0 + r, c = colof<G>(g, j);
      Pr[r * CW + j] = p.P0 != nullptr ? p.P0[((size_t)bh * D + row) * D + c] : (c == row ? 1.f : 0.f);
    }
  // the next block's keys and scalars travel in registers while the current block is walked
  float kr[Sh::KPT];
  float ra = 1.f, rr = 1.f, rq = 0.f;
  auto fetch = [&](int blk) {
    const int t0 = blk * kFB;
    load_keys<D>(p, tok0, t0, tid, kr);
    if (tid < kFB && t0 + tid < L) {
      const size_t ti = tok0 + t0 + tid;
      ra = p.a != nullptr ? p.a[ti] : 1.f, rr = p.r[ti], rq = p.qn != nullptr ? p.qn[ti] : p.qn_scalar;
    }
  };
  auto stash = [&](int buf) {
#pragma unroll
    for (int r = 0; r < Sh::KPT; ++r) (&kf[buf][0][0])[tid + Sh::NT * r] = kr[r];
    if (tid < kFB) sa[buf][tid] = ra, sr[buf][tid] = rr, sq[buf][tid] = rq;
  };
  fetch(0);
  stash(0);
  __syncthreads();
  if (nblk > 1) fetch(1);
  for (int blk = 0; blk < nblk; ++blk) {
    const int b = blk & 1, t0 = blk * kFB, n = min(kFB, L - t0);
    float* ck = p.ckpt + ((size_t)bh * nblk + blk) * D * D;
#pragma unroll
    for (int m = 0; m < Sh::NV; ++m)
      *slot<D>(ck, m, tid) = make_float4(Pr[4 * m], Pr[4 * m + 1], Pr[4 * m + 2], Pr[4 * m + 3]);
    for (int tt = 0; tt < n; ++tt) {
      float ui[R], s;
      cov_step<D>(Pr, kf[b][tt], us[tt & 1], part[tt & 1], sa[b][tt], sr[b][tt], sq[b][tt], tid, nullptr, ui, s);
      if (g == 0)  // (the backward's recompute checks s)
#pragma unroll
        for (int r = 0; r < R; ++r) p.gains[(tok0 + t0 + tt) * D + r0 + r] = ui[r] / s;
    }
    if (blk + 1 < nblk) {
      stash(b ^ 1);  // the other buffer was last read in block blk - 1, before this block's barriers
      __syncthreads();
      if (blk + 2 < nblk) fetch(blk + 2);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(4 * D, 1) full_cov_backward_kernel(FullBwdArgs p) {
  using Sh = FullBwdShape<D>;
  constexpr int R = Sh::R, G = Sh::G, CW = Sh::CW, NV = Sh::NV, NW = Sh::NW;
  // dynamic: [2][D * D] P before the token (thread order) | keys | u | dG | dk in, [kFB][D] fp32 each
  extern __shared__ __align__(16) float dyn[];
  float* pbuf = dyn;
  float(*kf)[D] = reinterpret_cast<float(*)[D]>(dyn + 2 * D * D);
  float(*ub)[D] = reinterpret_cast<float(*)[D]>(dyn + 2 * D * D + kFB * D);
  float(*gb)[D] = reinterpret_cast<float(*)[D]>(dyn + 2 * D * D + 2 * kFB * D);
  float(*dkb)[D] = reinterpret_cast<float(*)[D]>(dyn + 2 * D * D + 3 * kFB * D);
  __shared__ float sa[kFB], sr[kFB], sq[kFB], sda[kFB], ss[kFB];
  __shared__ __align__(16) float dus[2][D];
  __shared__ __align__(16) float part[2][3][NW], part2[2][2][NW], rpart[2][NW];
  const int tid = threadIdx.x, bh = blockIdx.x, L = p.L, lane = tid & 31, warp = tid >> 5;
  const int g = tid % G, r0 = (tid / G) * R;
  const bool row_lead = g == 0;
  const size_t tok0 = (size_t)bh * L;
  const int nblk = (L + kFB - 1) / kFB;
  float* scrP = p.scr_P + (size_t)bh * kFB * D * D;

  // M = dP_L + dP_L^T, and its trace
  float Mr[R * CW];
  float tr = 0.f;
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int j = 0; j < CW; ++j) {
      const size_t base = (size_t)bh * D * D;
      const int row = r0 + r, c = colof<G>(g, j);
      Mr[r * CW + j] =
          p.dP_L != nullptr ? p.dP_L[base + (size_t)row * D + c] + p.dP_L[base + (size_t)c * D + row] : 0.f;
      if (c == row) tr += Mr[r * CW + j];
    }
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) tr += __shfl_xor_sync(0xffffffffu, tr, o);
  if (lane == 0) rpart[0][warp] = tr;
  __syncthreads();
  float trM = sum_parts<NW>(rpart[0]);
  __syncthreads();

  for (int blk = nblk - 1; blk >= 0; --blk) {
    const int t0 = blk * kFB, n = min(kFB, L - t0);
    // ---------------------------------------------------------------- the block's inputs
    {
      // dG and the memory backward's dk rows (contiguous fp32, 16-byte chunks), then the keys and scalars
      const int chunks = n * D / 4;
      const float* gsrc = p.dgain + (tok0 + t0) * D;
      const float* ksrc = p.dk + (tok0 + t0) * D;
      for (int c = tid; c < chunks; c += Sh::NT) {
        async_copy16(&gb[0][0] + 4 * c, gsrc + 4 * c);
        async_copy16(&dkb[0][0] + 4 * c, ksrc + 4 * c);
      }
      async_commit();
      float kr[Sh::KPT];
      load_keys<D>(p, tok0, t0, tid, kr);
#pragma unroll
      for (int r = 0; r < Sh::KPT; ++r) (&kf[0][0])[tid + Sh::NT * r] = kr[r];
      if (tid < n) {
        const size_t ti = tok0 + t0 + tid;
        sa[tid] = p.a != nullptr ? p.a[ti] : 1.f, sr[tid] = p.r[ti];
        sq[tid] = p.qn != nullptr ? p.qn[ti] : p.qn_scalar, sda[tid] = p.da != nullptr ? p.da[ti] : 0.f;
      }
    }
    // ---------------------------------------------------------------- recompute the block's P, u, s
    {
      const float* ck = p.ckpt + ((size_t)bh * nblk + blk) * D * D;
      float Pr[R * CW];
#pragma unroll
      for (int m = 0; m < NV; ++m) {
        const float4 x = *slot<D>(const_cast<float*>(ck), m, tid);
        Pr[4 * m] = x.x, Pr[4 * m + 1] = x.y, Pr[4 * m + 2] = x.z, Pr[4 * m + 3] = x.w;
      }
      async_wait<0>();
      __syncthreads();
      for (int tt = 0; tt < n; ++tt) {
        float* sp = scrP + (size_t)tt * D * D;
#pragma unroll
        for (int m = 0; m < NV; ++m)
          *slot<D>(sp, m, tid) = make_float4(Pr[4 * m], Pr[4 * m + 1], Pr[4 * m + 2], Pr[4 * m + 3]);
        float ui[R], s;
        cov_step<D>(Pr, kf[tt], ub[tt], rpart[tt & 1], sa[tt], sr[tt], sq[tt], tid, p.status, ui, s);
        if (tid == 0) ss[tt] = s;
      }
      __syncthreads();  // ss and the scratch P are complete
    }
    // ---------------------------------------------------------------- the block in reverse
    auto fetch_P = [&](int tt) {  // each thread copies (and later reads) only its own slots
      float* dst = pbuf + (tt & 1) * D * D;
      const float* src = scrP + (size_t)tt * D * D;
#pragma unroll
      for (int m = 0; m < NV; ++m) async_copy16(slot<D>(dst, m, tid), slot<D>(const_cast<float*>(src), m, tid));
      async_commit();
    };
    fetch_P(n - 1);
    for (int tt = n - 1; tt >= 0; --tt) {
      const int b = tt & 1;
      const size_t ti = tok0 + t0 + tt;
      async_wait<0>();
      float Pp[R * CW];
#pragma unroll
      for (int m = 0; m < NV; ++m) {
        const float4 x = *slot<D>(pbuf + b * D * D, m, tid);
        Pp[4 * m] = x.x, Pp[4 * m + 1] = x.y, Pp[4 * m + 2] = x.z, Pp[4 * m + 3] = x.w;
      }
      if (tt > 0) fetch_P(tt - 1);
      const float at = sa[tt], qt = sq[tt], s = ss[tt], a2 = at * at, inv = 1.f / s;
      float ui[R], ki[R], dgi[R];
#pragma unroll
      for (int r = 0; r < R; ++r) ui[r] = ub[tt][r0 + r], ki[r] = kf[tt][r0 + r], dgi[r] = gb[tt][r0 + r];
      float mu4[R][4], pk4[R][4], mp4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int e = 0; e < 4; ++e) mu4[r][e] = pk4[r][e] = 0.f;
#pragma unroll
      for (int m = 0; m < Sh::NM; ++m) {
        const float4 u4 = vec4<G>(ub[tt], m, g), k4 = vec4<G>(kf[tt], m, g);
        const float uu[4] = {u4.x, u4.y, u4.z, u4.w}, kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int x = r * CW + 4 * m + e;
            mu4[r][e] = fmaf(Mr[x], uu[e], mu4[r][e]);
            pk4[r][e] = fmaf(Pp[x], kk[e], pk4[r][e]);
            mp4[e] = fmaf(Mr[x], Pp[x], mp4[e]);
          }
      }
      float Mu[R], Pk[R], x0 = 0.f, x1 = 0.f;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        Mu[r] = group_sum<G>((mu4[r][0] + mu4[r][1]) + (mu4[r][2] + mu4[r][3]));
        Pk[r] = group_sum<G>((pk4[r][0] + pk4[r][1]) + (pk4[r][2] + pk4[r][3]));
        if (row_lead) x0 = fmaf(dgi[r], ui[r], x0), x1 = fmaf(ui[r], Mu[r], x1);
      }
      float x2 = (mp4[0] + mp4[1]) + (mp4[2] + mp4[3]);
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        x0 += __shfl_xor_sync(0xffffffffu, x0, o);
        x1 += __shfl_xor_sync(0xffffffffu, x1, o);
        x2 += __shfl_xor_sync(0xffffffffu, x2, o);
      }
      if (lane == 0) part[b][0][warp] = x0, part[b][1][warp] = x1, part[b][2][warp] = x2;
      __syncthreads();
      const float dgu = sum_parts<NW>(part[b][0]), uMu = sum_parts<NW>(part[b][1]), MPs = sum_parts<NW>(part[b][2]);
      const float ds = (0.5f * uMu - dgu) * inv * inv;
      float dui[R], y0 = 0.f, y1 = 0.f;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        dui[r] = (dgi[r] - Mu[r]) * inv + ds * ki[r];
        if (row_lead) {
          dus[b][r0 + r] = dui[r];
          y0 = fmaf(dui[r], Pk[r], y0), y1 = fmaf(dui[r], ki[r], y1);
        }
      }
#pragma unroll
      for (int o = G; o < 32; o <<= 1) {
        y0 += __shfl_xor_sync(0xffffffffu, y0, o);
        y1 += __shfl_xor_sync(0xffffffffu, y1, o);
      }
      if (lane == 0) part2[b][0][warp] = y0, part2[b][1][warp] = y1;
      __syncthreads();
      const float duPk = sum_parts<NW>(part2[b][0]), duk = sum_parts<NW>(part2[b][1]);
      // P du and the update of M in one pass over this thread's columns of du and k
      float pd4[R][4];
#pragma unroll
      for (int r = 0; r < R; ++r) pd4[r][0] = pd4[r][1] = pd4[r][2] = pd4[r][3] = 0.f;
#pragma unroll
      for (int m = 0; m < Sh::NM; ++m) {
        const float4 k4 = vec4<G>(kf[tt], m, g), d4 = vec4<G>(dus[b], m, g);
        const float kk[4] = {k4.x, k4.y, k4.z, k4.w}, dd[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int x = r * CW + 4 * m + e;
            pd4[r][e] = fmaf(Pp[x], dd[e], pd4[r][e]);
            Mr[x] = a2 * (Mr[x] + fmaf(dui[r], kk[e], ki[r] * dd[e]));
          }
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float Pdu = group_sum<G>((pd4[r][0] + pd4[r][1]) + (pd4[r][2] + pd4[r][3]));
        if (row_lead) p.dk[ti * D + r0 + r] = dkb[tt][r0 + r] + ds * ui[r] + a2 * Pdu + qt * dui[r];
      }
      if (tid == 0) {
        p.dr[ti] = ds;
        p.dqn[ti] = 0.5f * trM + duk;
        if (p.da != nullptr) p.da[ti] = sda[tt] + 2.f * at * (0.5f * MPs + duPk);
      }
      trM = a2 * (trM + 2.f * duk);
    }
    __syncthreads();  // the block's buffers are free for the next block
  }
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int j = 0; j < CW; ++j) p.dP0[((size_t)bh * D + r0 + r) * D + colof<G>(g, j)] = 0.5f * Mr[r * CW + j];
}

template <int D>
cudaError_t launch_full_typed(const FullBwdArgs& args, int BH, bool backward, cudaStream_t stream) {
  if (!backward) {
    if (args.L <= 0) return cudaSuccess;
    full_cov_forward_kernel<D><<<BH, 4 * D, 0, stream>>>(args);
    return cudaGetLastError();
  }
  const int smem = (2 * D * D + 4 * kFB * D) * 4;
  cudaError_t e = cudaFuncSetAttribute(full_cov_backward_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  full_cov_backward_kernel<D><<<BH, 4 * D, smem, stream>>>(args);
  return cudaGetLastError();
}

cudaError_t launch_full(const FullBwdArgs& args, int BH, bool backward, cudaStream_t stream) {
  if (BH <= 0) return cudaSuccess;
  switch (args.d) {
    case 16: return launch_full_typed<16>(args, BH, backward, stream);
    case 32: return launch_full_typed<32>(args, BH, backward, stream);
    case 64: return launch_full_typed<64>(args, BH, backward, stream);
    case 128: return launch_full_typed<128>(args, BH, backward, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

size_t full_backward_scratch_bytes(int BH, int L, int d) {
  const size_t nblk = ((size_t)L + kFB - 1) / kFB, dd = (size_t)d * d;
  auto r256 = [](size_t x) { return (x + 255) / 256 * 256; };
  return r256((size_t)BH * nblk * dd * 4) + r256((size_t)BH * kFB * dd * 4);
}

void full_backward_bind_scratch(FullBwdArgs& args, void* scratch, int BH) {
  const size_t nblk = ((size_t)args.L + kFB - 1) / kFB, dd = (size_t)args.d * args.d;
  auto r256 = [](size_t x) { return (x + 255) / 256 * 256; };
  char* s = static_cast<char*>(scratch);
  args.ckpt = reinterpret_cast<float*>(s);
  s += r256((size_t)BH * nblk * dd * 4);
  args.scr_P = reinterpret_cast<float*>(s);
}

cudaError_t launch_full_cov_forward(const FullBwdArgs& args, int BH, cudaStream_t stream) {
  return launch_full(args, BH, false, stream);
}

cudaError_t launch_full_cov_backward(const FullBwdArgs& args, int BH, cudaStream_t stream) {
  return launch_full(args, BH, true, stream);
}

}  // namespace kdn
