// Per-token (sequential) scan kernels on the fp32 CUDA cores.
//
// These are the exact token-by-token recurrences, one CTA per head with the
// state held in registers; they serve every shape the library accepts and are
// the reference the chunked tensor-core kernels are tested against.
//
// S-side (all variants), per token t with gain g_t
//   (A Hippocampus for Linear Attention, section 3.3 Eq. (5)-(6), section 3.5):
//     y_k = S^T k_t, y_q = S^T q_t                 (one reduction round)
//     e_t = v_t - a_t y_k
//     o_t = S_t^T q_t = a_t y_q + (g_t . q_t) e_t
//     S  <- a_t S + g_t e_t^T
//     m_t = ||g_t|| ||e_t||
// Covariance side (Kalman Delta Networks, Abstract; DeltaNet-PC Eq. (7)):
//     full  P^- = a^2 P + Qn I, u = P^- k, s = k.u + r, g = u / s,
//           P <- P^- - u u^T / s
//     diag  p^- = a^2 p + Qn, s = sum p^- k^2 + r, g = p^- k / s,
//           p <- p^- r / (r + p^- k^2)
#include "common.cuh"
#include "kernels.h"

namespace kdn {

constexpr int kTokBlock = 16;  // tokens staged in shared memory at a time

// Raw inputs of one token block in shared memory (the per-token kernel's two-stage ring, copied
// asynchronously one block ahead): k, q ([16][DK], bf16 or fp32 as given), v ([16][DV]), gains ([16][DK] fp32,
// Kalman), a and beta ([16] each).  Sized for fp32 inputs.
template <int DK, int DV, bool kGains>
struct RawStage {
  static constexpr int K = 0, Q = K + kTokBlock * DK * 4, V = Q + kTokBlock * DK * 4, G = V + kTokBlock * DV * 4;
  static constexpr int A = G + (kGains ? kTokBlock * DK * 4 : 0), B = A + kTokBlock * 4;
  static constexpr int BYTES = B + kTokBlock * 4;
};

template <int DK, int DV, bool kGainsFromWs>
__global__ void __launch_bounds__(RowBlockLayout<DK, DV>::kThreads) seq_scan_kernel(SeqScanArgs args) {
  using Lay = RowBlockLayout<DK, DV>;
  constexpr int NT = Lay::kThreads, CG = Lay::kColGroups, RG = Lay::kRowGroups, RPT = Lay::kRowsPerThread;
  constexpr int NW = NT / 32;
  constexpr int DVW = (DV + 31) / 32 * 32;
  static_assert(NT >= DVW, "phase B needs whole warps over d_v");

  __shared__ float k_s[kTokBlock][DK], q_s[kTokBlock][DK], g_s[kTokBlock][DK];
  __shared__ float v_s[kTokBlock][DV];
  __shared__ float a_s[kTokBlock], b_s[kTokBlock], gq_s[kTokBlock], gn_s[kTokBlock];
  __shared__ __align__(16) float red[RG][2][DV];
  __shared__ float e_s[DV];
  __shared__ float ered[DVW / 32];

  const int bh = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cg = tid % CG, rg = tid / CG;
  const int L = args.L;
  const size_t tok0 = (size_t)bh * L;

  float S[RPT][4];
  float* Sg = args.S + (size_t)bh * DK * DV;
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const float4 x = *reinterpret_cast<const float4*>(Sg + (size_t)(rg + i * RG) * DV + cg * 4);
    S[i][0] = x.x, S[i][1] = x.y, S[i][2] = x.z, S[i][3] = x.w;
  }

  // the raw inputs of block b + 1 are copied while block b runs
  using RS = RawStage<DK, DV, kGainsFromWs>;
  extern __shared__ __align__(16) uint8_t raw[];
  const int es = args.in_dtype == kBF16 ? 2 : 4;
  const int nblk = (L + kTokBlock - 1) / kTokBlock;
  auto issue = [&](int blk) {
    if (blk < nblk) {
      const int t0 = blk * kTokBlock, nt = min(kTokBlock, L - t0);
      uint8_t* st = raw + (blk & 1) * RS::BYTES;
      async_copy_rows(st + RS::K, static_cast<const uint8_t*>(args.k) + (tok0 + t0) * DK * es, nt * DK * es, tid, NT);
      async_copy_rows(st + RS::Q, static_cast<const uint8_t*>(args.q) + (tok0 + t0) * DK * es, nt * DK * es, tid, NT);
      async_copy_rows(st + RS::V, static_cast<const uint8_t*>(args.v) + (tok0 + t0) * DV * es, nt * DV * es, tid, NT);
      if constexpr (kGainsFromWs) async_copy_rows(st + RS::G, args.gains + (tok0 + t0) * DK, nt * DK * 4, tid, NT);
      if (tid < nt) {
        float* sa_ = reinterpret_cast<float*>(st + RS::A);
        float* sb_ = reinterpret_cast<float*>(st + RS::B);
        if (args.a != nullptr) async_copy4(sa_ + tid, args.a + tok0 + t0 + tid); else sa_[tid] = 1.f;
        if (!kGainsFromWs) async_copy4(sb_ + tid, args.beta + tok0 + t0 + tid); else sb_[tid] = 0.f;
      }
    }
    async_commit();
  };
  issue(0);

  const int nck = args.S_ckpt != nullptr ? (L + args.ckpt_every - 1) / args.ckpt_every : 0;
  for (int t0 = 0; t0 < L; t0 += kTokBlock) {
    const int nt = min(kTokBlock, L - t0);
    const int blk = t0 / kTokBlock;
    if (nck > 0 && t0 % args.ckpt_every == 0) {  // the state entering this checkpoint chunk
      float* Sc = args.S_ckpt + ((size_t)bh * nck + t0 / args.ckpt_every) * DK * DV;
#pragma unroll
      for (int i = 0; i < RPT; ++i)
        *reinterpret_cast<float4*>(Sc + (size_t)(rg + i * RG) * DV + cg * 4) =
            make_float4(S[i][0], S[i][1], S[i][2], S[i][3]);
    }
    issue(blk + 1);
    async_wait<1>();
    __syncthreads();  // this block's raw inputs are in; the previous block's staged floats are no longer read
    {
      const uint8_t* st = raw + (blk & 1) * RS::BYTES;
      auto elem = [&](int off, int idx) {
        return args.in_dtype == kBF16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(st + off)[idx])
                                      : reinterpret_cast<const float*>(st + off)[idx];
      };
      for (int idx = tid; idx < nt * DK; idx += NT) {
        const int j = idx / DK, i = idx % DK;
        k_s[j][i] = elem(RS::K, idx);
        q_s[j][i] = elem(RS::Q, idx);
        if constexpr (kGainsFromWs) g_s[j][i] = reinterpret_cast<const float*>(st + RS::G)[idx];
      }
      for (int idx = tid; idx < nt * DV; idx += NT) v_s[idx / DV][idx % DV] = elem(RS::V, idx);
      for (int j = tid; j < nt; j += NT) {
        a_s[j] = reinterpret_cast<const float*>(st + RS::A)[j];
        b_s[j] = reinterpret_cast<const float*>(st + RS::B)[j];
      }
    }
    __syncthreads();
    for (int j = warp; j < nt; j += NW) {
      float sq = 0.f, sn = 0.f;
      for (int i = lane; i < DK; i += 32) {
        const float g = kGainsFromWs ? g_s[j][i] : b_s[j] * k_s[j][i];
        sq = fmaf(g, q_s[j][i], sq);
        sn = fmaf(g, g, sn);
      }
      sq = warp_sum(sq);
      sn = warp_sum(sn);
      if (lane == 0) gq_s[j] = sq, gn_s[j] = sn;
    }
    __syncthreads();

    for (int j = 0; j < nt; ++j) {
      const float a = a_s[j];
      // phase A: partial S^T k and S^T q over this thread's rows
      float pk[4] = {0.f, 0.f, 0.f, 0.f}, pq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const int row = rg + i * RG;
        const float kr = k_s[j][row], qr = q_s[j][row];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          pk[c] = fmaf(S[i][c], kr, pk[c]);
          pq[c] = fmaf(S[i][c], qr, pq[c]);
        }
      }
      *reinterpret_cast<float4*>(&red[rg][0][cg * 4]) = make_float4(pk[0], pk[1], pk[2], pk[3]);
      *reinterpret_cast<float4*>(&red[rg][1][cg * 4]) = make_float4(pq[0], pq[1], pq[2], pq[3]);
      __syncthreads();
      // phase B: residual, output, residual norm
      if (tid < DVW) {
        float e = 0.f;
        if (tid < DV) {
          float yk = 0.f, yq = 0.f;
#pragma unroll
          for (int r = 0; r < RG; ++r) yk += red[r][0][tid], yq += red[r][1][tid];
          e = v_s[j][tid] - a * yk;
          if (args.o != nullptr)
            store_elem(args.o, (tok0 + t0 + j) * DV + tid, fmaf(a, yq, gq_s[j] * e), args.out_dtype);
          e_s[tid] = e;
        }
        const float es = warp_sum(e * e);
        if (lane == 0) ered[warp] = es;
      }
      __syncthreads();
      // phase C: rank-1 write
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const int row = rg + i * RG;
        const float gr = kGainsFromWs ? g_s[j][row] : b_s[j] * k_s[j][row];
#pragma unroll
        for (int c = 0; c < 4; ++c) S[i][c] = fmaf(a, S[i][c], gr * e_s[cg * 4 + c]);
      }
      if (tid == 0 && (args.m != nullptr || args.enorm != nullptr)) {
        float es = 0.f;
#pragma unroll
        for (int w = 0; w < DVW / 32; ++w) es += ered[w];
        if (args.m != nullptr) args.m[tok0 + t0 + j] = sqrtf(gn_s[j]) * sqrtf(es);
        if (args.enorm != nullptr) args.enorm[tok0 + t0 + j] = sqrtf(es);
      }
    }
  }
  async_wait<0>();
#pragma unroll
  for (int i = 0; i < RPT; ++i)
    *reinterpret_cast<float4*>(Sg + (size_t)(rg + i * RG) * DV + cg * 4) = make_float4(S[i][0], S[i][1], S[i][2], S[i][3]);
}

// Full-covariance Riccati recursion, one token at a time, one CTA per head.  Four
// consecutive threads share column c of P (symmetric, so P^- k is a column dot
// product); each holds d_k/4 of its rows in registers.  The accumulated process
// noise is kept as a scalar offset, P = Pt + c I with c <- a^2 c + Qn, so the
// diagonal is never touched: u = P^- k = a^2 Pt k + c k, Pt <- a^2 Pt - u u^T / s.
// One block barrier per token (u and the pieces of s = k.u + r go through
// double-buffered shared slots).  Shared vectors are stored with a 4-float skew
// per 32 floats so that the four row segments of a column sit in distinct banks.
__device__ __forceinline__ int skew32(int x) { return x + ((x >> 5) << 2); }

template <int DK>
__global__ void __launch_bounds__(4 * DK) kalman_full_gains_kernel(GainArgs args) {
  constexpr int NT = 4 * DK, RP = DK / 4, NW = NT / 32;
  constexpr int DKS = (DK + DK / 8 + 3) / 4 * 4;  // skewed width, rows 16-byte aligned
  __shared__ __align__(16) float k_s[kTokBlock][DKS];
  __shared__ float a_s[kTokBlock], qn_s[kTokBlock], r_s[kTokBlock];
  __shared__ __align__(16) float u_s[2][DKS];
  __shared__ float red[2][NW];

  const int bh = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int col = tid >> 2, part = tid & 3, r0 = part * RP;
  const int L = args.L;
  const size_t tok0 = (size_t)bh * L;

  float Pc[RP];  // Pt[r0 + i][col]
  const float* Prow = args.P + (size_t)bh * DK * DK + (size_t)col * DK + r0;
#pragma unroll
  for (int i = 0; i < RP; i += 4) {
    const float4 x = *reinterpret_cast<const float4*>(Prow + i);
    Pc[i] = x.x, Pc[i + 1] = x.y, Pc[i + 2] = x.z, Pc[i + 3] = x.w;
  }
  float cI = 0.f;  // P = Pt + cI * I
  const int sr0 = skew32(r0), scol = skew32(col);

  int par = 0;
  for (int t0 = 0; t0 < L; t0 += kTokBlock) {
    const int nt = min(kTokBlock, L - t0);
    __syncthreads();
    for (int idx = tid; idx < nt * DK; idx += NT) {
      const int j = idx / DK, i = idx % DK;
      k_s[j][skew32(i)] = load_elem(args.k, (tok0 + t0 + j) * DK + i, args.in_dtype);
    }
    for (int j = tid; j < nt; j += NT) {
      const size_t tk = tok0 + t0 + j;
      a_s[j] = args.a ? args.a[tk] : 1.f;
      qn_s[j] = args.qn ? args.qn[tk] : args.qn_scalar;
      r_s[j] = args.r[tk];
    }
    __syncthreads();
    for (int j = 0; j < nt; ++j) {
      const float a2 = a_s[j] * a_s[j];
      cI = fmaf(a2, cI, qn_s[j]);
      float v0 = 0.f, v1 = 0.f, v2 = 0.f, v3 = 0.f;
#pragma unroll
      for (int i = 0; i < RP; i += 4) {  // RP is a multiple of 4 and a segment never crosses a skew boundary
        const float4 k4 = *reinterpret_cast<const float4*>(&k_s[j][sr0 + i]);
        v0 = fmaf(Pc[i], k4.x, v0);
        v1 = fmaf(Pc[i + 1], k4.y, v1);
        v2 = fmaf(Pc[i + 2], k4.z, v2);
        v3 = fmaf(Pc[i + 3], k4.w, v3);
      }
      float v = (v0 + v1) + (v2 + v3);
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      const float kc = k_s[j][scol];
      v = fmaf(a2, v, cI * kc);  // u_col
      float sp = (part == 0) ? kc * v : 0.f;
      sp = warp_sum(sp);
      if (part == 0) u_s[par][scol] = v;
      if (lane == 0) red[par][warp] = sp;
      __syncthreads();
      float s = r_s[j];
#pragma unroll
      for (int w = 0; w < NW; ++w) s += red[par][w];
      if (tid == 0 && !(s > 0.f && isfinite(s))) raise_status(args.status, kStatusNumeric);
      const float gcol = v / s;
      if (part == 0) args.gains[(tok0 + t0 + j) * DK + col] = gcol;
#pragma unroll
      for (int i = 0; i < RP; i += 4) {
        const float4 u4 = *reinterpret_cast<const float4*>(&u_s[par][sr0 + i]);
        Pc[i] = fmaf(-u4.x, gcol, a2 * Pc[i]);
        Pc[i + 1] = fmaf(-u4.y, gcol, a2 * Pc[i + 1]);
        Pc[i + 2] = fmaf(-u4.z, gcol, a2 * Pc[i + 2]);
        Pc[i + 3] = fmaf(-u4.w, gcol, a2 * Pc[i + 3]);
      }
      par ^= 1;
    }
  }
  if (col >= r0 && col < r0 + RP) {
#pragma unroll
    for (int i = 0; i < RP; ++i)
      if (r0 + i == col) Pc[i] += cI;
  }
  float* Pw = args.P + (size_t)bh * DK * DK + (size_t)col * DK + r0;
#pragma unroll
  for (int i = 0; i < RP; i += 4) *reinterpret_cast<float4*>(Pw + i) = make_float4(Pc[i], Pc[i + 1], Pc[i + 2], Pc[i + 3]);
}

// One warp per head; the p recursion is sequential in t and cheap.
template <int DK>
__global__ void __launch_bounds__(128) kalman_diag_gains_kernel(GainArgs args) {
  constexpr int PER = (DK + 31) / 32;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (bh >= args.BH) return;
  const int L = args.L;
  const size_t tok0 = (size_t)bh * L;
  float p[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int c = lane + 32 * i;
    p[i] = c < DK ? args.p[(size_t)bh * DK + c] : 0.f;
  }
  for (int t = 0; t < L; ++t) {
    const size_t tk = tok0 + t;
    const float a = args.a ? args.a[tk] : 1.f;
    const float qn = args.qn ? args.qn[tk] : args.qn_scalar;
    const float r = args.r[tk];
    float kk[PER], pp[PER], part = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int c = lane + 32 * i;
      kk[i] = c < DK ? load_elem(args.k, tk * DK + c, args.in_dtype) : 0.f;
      pp[i] = c < DK ? fmaf(a * a, p[i], qn) : 0.f;
      part = fmaf(pp[i] * kk[i], kk[i], part);
    }
    const float s = warp_sum(part) + r;
    if (lane == 0 && !(s > 0.f && isfinite(s))) raise_status(args.status, kStatusNumeric);
    const float inv_s = 1.f / s;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int c = lane + 32 * i;
      if (c < DK) {
        args.gains[tk * DK + c] = pp[i] * kk[i] * inv_s;
        p[i] = pp[i] * r / fmaf(pp[i] * kk[i], kk[i], r);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int c = lane + 32 * i;
    if (c < DK) args.p[(size_t)bh * DK + c] = p[i];
  }
}

#define KDN_DIMS_SWITCH(D, NAME, ...)         \
  switch (D) {                                \
    case 16: { constexpr int NAME = 16; __VA_ARGS__; } break;   \
    case 32: { constexpr int NAME = 32; __VA_ARGS__; } break;   \
    case 64: { constexpr int NAME = 64; __VA_ARGS__; } break;   \
    case 128: { constexpr int NAME = 128; __VA_ARGS__; } break; \
    default: return cudaErrorInvalidValue;    \
  }

cudaError_t launch_seq_scan(int dk, int dv, const SeqScanArgs& args, cudaStream_t stream) {
  if (args.BH <= 0 || args.L <= 0) return cudaSuccess;
  KDN_DIMS_SWITCH(dk, DK, KDN_DIMS_SWITCH(dv, DV, {
    constexpr int NT = RowBlockLayout<DK, DV>::kThreads;
    if (args.gains != nullptr) {
      constexpr int smem = 2 * RawStage<DK, DV, true>::BYTES;
      cudaError_t e = cudaFuncSetAttribute(seq_scan_kernel<DK, DV, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      seq_scan_kernel<DK, DV, true><<<args.BH, NT, smem, stream>>>(args);
    } else {
      constexpr int smem = 2 * RawStage<DK, DV, false>::BYTES;
      cudaError_t e = cudaFuncSetAttribute(seq_scan_kernel<DK, DV, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      seq_scan_kernel<DK, DV, false><<<args.BH, NT, smem, stream>>>(args);
    }
  }));
  return cudaGetLastError();
}

cudaError_t launch_kalman_full_gains(int dk, const GainArgs& args, cudaStream_t stream) {
  if (args.BH <= 0 || args.L <= 0) return cudaSuccess;
  KDN_DIMS_SWITCH(dk, DK, { kalman_full_gains_kernel<DK><<<args.BH, 4 * DK, 0, stream>>>(args); });
  return cudaGetLastError();
}

cudaError_t launch_kalman_diag_gains(int dk, const GainArgs& args, cudaStream_t stream) {
  if (args.BH <= 0 || args.L <= 0) return cudaSuccess;
  KDN_DIMS_SWITCH(dk, DK, { kalman_diag_gains_kernel<DK><<<(args.BH + 3) / 4, 128, 0, stream>>>(args); });
  return cudaGetLastError();
}

}  // namespace kdn
