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
// One CTA of 4 d threads per head: thread (i, q) = (tid / 4, tid % 4) holds row i of P (and of M) at the d/4
// columns 16 m + 4 q + e (e < 4), so a matrix-vector product is d/4 multiply-adds per thread and a reduction
// over four lanes, and the four threads of a row read a broadcast vector as four adjacent float4, free of
// bank conflicts (with columns q d/4 .. per thread the four quarters would sit on the same banks).  Both
// kernels go through the tokens in blocks of kFB, each block's inputs staged in shared memory before it is
// walked (the forward loads the next block into registers while it walks the current one), so no global
// load sits on a token's serial path.  The forward keeps P at every block start;
// the backward recomputes each block's P before every token (to global scratch, in the threads' own float4
// order; u and s stay in shared memory), then walks the block in reverse with that P streamed back through a
// two-slot cp.async buffer, each thread copying and reading only its own slots.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace kdn {

namespace {

constexpr int kFB = 32;  // tokens per block: inputs staged per block, P checkpointed and recomputed per block

template <int D>
struct FullBwdShape {
  static constexpr int NT = 4 * D, NW = NT / 32, CW = D / 4, NV = CW / 4;  // NV float4 per thread per matrix
  static constexpr int KPT = kFB * D / NT;  // block elements per thread when a [kFB, D] block is staged
};

// Thread tid's slot m of a d x d matrix held in thread order: float4 m * NT + tid.
template <int D>
__device__ __forceinline__ float4* slot(float* base, int m, int tid) {
  return reinterpret_cast<float4*>(base) + (size_t)m * FullBwdShape<D>::NT + tid;
}

// Column of register j of thread quarter q, and that thread's float4 m of a d-vector in shared memory.
__device__ __forceinline__ int colof(int q, int j) { return 16 * (j >> 2) + 4 * q + (j & 3); }
__device__ __forceinline__ float4 vec4(const float* v, int m, int q) {
  return reinterpret_cast<const float4*>(v)[4 * m + q];
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

// One forward token of P held by the calling thread: P <- P^- - u u^T / s.  kv holds the token's key (fp32),
// us receives u (it is also this token's broadcast slot), part the warp partial sums.  Returns u_i and s;
// one __syncthreads.
template <int D>
__device__ __forceinline__ void cov_step(float (&Pr)[D / 4], const float* kv, float* us, float* part, float at,
                                         float rt, float qt, int tid, unsigned* status, float& ui, float& s) {
  using Sh = FullBwdShape<D>;
  const int i = tid >> 2, q = tid & 3, lane = tid & 31, warp = tid >> 5;
  const float a2 = at * at;
  float d4[4] = {0.f, 0.f, 0.f, 0.f};  // four partial sums keep the dependent chain d / 16 long
#pragma unroll
  for (int m = 0; m < Sh::NV; ++m) {
    const float4 k4 = vec4(kv, m, q);
    const float kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = 4 * m + e;
      Pr[j] = fmaf(a2, Pr[j], colof(q, j) == i ? qt : 0.f);
      d4[e] = fmaf(Pr[j], kk[e], d4[e]);
    }
  }
  float dot = (d4[0] + d4[1]) + (d4[2] + d4[3]);
  dot += __shfl_xor_sync(0xffffffffu, dot, 1);
  dot += __shfl_xor_sync(0xffffffffu, dot, 2);
  ui = dot;
  float ku = (tid & 3) == 0 ? kv[i] * ui : 0.f;
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) ku += __shfl_xor_sync(0xffffffffu, ku, o);
  if (lane == 0) part[warp] = ku;
  if ((tid & 3) == 0) us[i] = ui;
  __syncthreads();
  s = rt + sum_parts<Sh::NW>(part);
  if (tid == 0 && status != nullptr && !(s > 0.f && isfinite(s))) raise_status(status, kStatusNumeric);
  const float f = ui / s;
#pragma unroll
  for (int m = 0; m < Sh::NV; ++m) {
    const float4 u4 = vec4(us, m, q);
    Pr[4 * m] = fmaf(-f, u4.x, Pr[4 * m]), Pr[4 * m + 1] = fmaf(-f, u4.y, Pr[4 * m + 1]);
    Pr[4 * m + 2] = fmaf(-f, u4.z, Pr[4 * m + 2]), Pr[4 * m + 3] = fmaf(-f, u4.w, Pr[4 * m + 3]);
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
  const int tid = threadIdx.x, bh = blockIdx.x, L = p.L;
  const int i = tid >> 2, q = tid & 3;
  const size_t tok0 = (size_t)bh * L;
  const int nblk = (L + kFB - 1) / kFB;
  float Pr[Sh::CW];
#pragma unroll
  for (int j = 0; j < Sh::CW; ++j)
    Pr[j] = p.P0 != nullptr ? p.P0[((size_t)bh * D + i) * D + colof(q, j)] : (colof(q, j) == i ? 1.f : 0.f);
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
      float ui, s;
      cov_step<D>(Pr, kf[b][tt], us[tt & 1], part[tt & 1], sa[b][tt], sr[b][tt], sq[b][tt], tid, nullptr, ui, s);
      if ((tid & 3) == 0) p.gains[(tok0 + t0 + tt) * D + i] = ui / s;  // (the backward's recompute checks s)
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
  constexpr int CW = Sh::CW, NV = Sh::NV, NW = Sh::NW;
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
  const int i = tid >> 2, q = tid & 3;
  const bool row_lead = q == 0;
  const size_t tok0 = (size_t)bh * L;
  const int nblk = (L + kFB - 1) / kFB;
  float* scrP = p.scr_P + (size_t)bh * kFB * D * D;

  // M = dP_L + dP_L^T, and its trace
  float Mr[CW];
  float tr = 0.f;
#pragma unroll
  for (int j = 0; j < CW; ++j) {
    const size_t base = (size_t)bh * D * D;
    const int c = colof(q, j);
    Mr[j] = p.dP_L != nullptr ? p.dP_L[base + (size_t)i * D + c] + p.dP_L[base + (size_t)c * D + i] : 0.f;
    if (c == i) tr = Mr[j];
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
      float Pr[CW];
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
        float ui, s;
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
      float Pp[CW];
#pragma unroll
      for (int m = 0; m < NV; ++m) {
        const float4 x = *slot<D>(pbuf + b * D * D, m, tid);
        Pp[4 * m] = x.x, Pp[4 * m + 1] = x.y, Pp[4 * m + 2] = x.z, Pp[4 * m + 3] = x.w;
      }
      if (tt > 0) fetch_P(tt - 1);
      const float at = sa[tt], qt = sq[tt], s = ss[tt], a2 = at * at, inv = 1.f / s;
      const float ui = ub[tt][i], ki = kf[tt][i], dgi = gb[tt][i];
      float mu4[4] = {0.f, 0.f, 0.f, 0.f}, pk4[4] = {0.f, 0.f, 0.f, 0.f}, mp4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int m = 0; m < NV; ++m) {
        const float4 u4 = vec4(ub[tt], m, q), k4 = vec4(kf[tt], m, q);
        const float uu[4] = {u4.x, u4.y, u4.z, u4.w}, kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 4 * m + e;
          mu4[e] = fmaf(Mr[j], uu[e], mu4[e]);
          pk4[e] = fmaf(Pp[j], kk[e], pk4[e]);
          mp4[e] = fmaf(Mr[j], Pp[j], mp4[e]);
        }
      }
      float Mu = (mu4[0] + mu4[1]) + (mu4[2] + mu4[3]), Pk = (pk4[0] + pk4[1]) + (pk4[2] + pk4[3]);
      const float MP = (mp4[0] + mp4[1]) + (mp4[2] + mp4[3]);
      Mu += __shfl_xor_sync(0xffffffffu, Mu, 1);
      Mu += __shfl_xor_sync(0xffffffffu, Mu, 2);
      Pk += __shfl_xor_sync(0xffffffffu, Pk, 1);
      Pk += __shfl_xor_sync(0xffffffffu, Pk, 2);
      // every lane of a row holds u_i and the reduced Mu, so the row terms take each lane's quarter
      float x0 = 0.25f * dgi * ui, x1 = 0.25f * ui * Mu, x2 = MP;
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
      const float dui = (dgi - Mu) * inv + ds * ki;
      if (row_lead) dus[b][i] = dui;
      float y0 = row_lead ? dui * Pk : 0.f, y1 = row_lead ? dui * ki : 0.f;
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        y0 += __shfl_xor_sync(0xffffffffu, y0, o);
        y1 += __shfl_xor_sync(0xffffffffu, y1, o);
      }
      if (lane == 0) part2[b][0][warp] = y0, part2[b][1][warp] = y1;
      __syncthreads();
      const float duPk = sum_parts<NW>(part2[b][0]), duk = sum_parts<NW>(part2[b][1]);
      float pd4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int m = 0; m < NV; ++m) {
        const float4 d4 = vec4(dus[b], m, q);
        pd4[0] = fmaf(Pp[4 * m], d4.x, pd4[0]), pd4[1] = fmaf(Pp[4 * m + 1], d4.y, pd4[1]);
        pd4[2] = fmaf(Pp[4 * m + 2], d4.z, pd4[2]), pd4[3] = fmaf(Pp[4 * m + 3], d4.w, pd4[3]);
      }
      float Pdu = (pd4[0] + pd4[1]) + (pd4[2] + pd4[3]);
      Pdu += __shfl_xor_sync(0xffffffffu, Pdu, 1);
      Pdu += __shfl_xor_sync(0xffffffffu, Pdu, 2);
      if (row_lead) p.dk[ti * D + i] = dkb[tt][i] + ds * ui + a2 * Pdu + qt * dui;
      if (tid == 0) {
        p.dr[ti] = ds;
        p.dqn[ti] = 0.5f * trM + duk;
        if (p.da != nullptr) p.da[ti] = sda[tt] + 2.f * at * (0.5f * MPs + duPk);
      }
#pragma unroll
      for (int m = 0; m < NV; ++m) {
        const float4 k4 = vec4(kf[tt], m, q), d4 = vec4(dus[b], m, q);
        Mr[4 * m] = a2 * (Mr[4 * m] + fmaf(dui, k4.x, ki * d4.x));
        Mr[4 * m + 1] = a2 * (Mr[4 * m + 1] + fmaf(dui, k4.y, ki * d4.y));
        Mr[4 * m + 2] = a2 * (Mr[4 * m + 2] + fmaf(dui, k4.z, ki * d4.z));
        Mr[4 * m + 3] = a2 * (Mr[4 * m + 3] + fmaf(dui, k4.w, ki * d4.w));
      }
      trM = a2 * (trM + 2.f * duk);
    }
    __syncthreads();  // the block's buffers are free for the next block
  }
#pragma unroll
  for (int j = 0; j < CW; ++j) p.dP0[((size_t)bh * D + i) * D + colof(q, j)] = 0.5f * Mr[j];
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
