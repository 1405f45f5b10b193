// Chunked scan on the sm_100a tensor cores (tcgen05 + TMEM + TMA), d_k = d_v = 64.  (d = 128 runs the
// warp-specialised kernel of chunk_scan_ws.cu; the host entry below dispatches both.)
//
// One CTA per head walks the sequence in chunks of C = 64 tokens.  Within a
// chunk, with A_i = prod_{m<=i} a_m and Gam_ij = A_i / A_j (i >= j), the
// token-by-token recurrence S_t = a_t S_{t-1} + g_t e_t^T,
// e_t = v_t - a_t S_{t-1}^T k_t (A Hippocampus for Linear Attention, section
// 3.3 Eq. (5) and section 3.5) is exactly the generalised WY / UT form
//
//   (I + N) E = R,    N = strict_lower((K G^T) o Gam),   R = V - diag(A) K S0
//   O   = diag(A) Q S0 + ((Q G^T) o Gam o lower) E
//   S_C = A_C S0 + G^T diag(A_C / A_j) E,      m_j = ||g_j|| ||e_j||
//
// where the rows g_j of G are the gains: beta_j k_j for the delta rule, or the
// diagonal-Kalman gains p^-_j o k_j / s_j (Kalman Delta Networks, Abstract:
// per-coordinate mean-field projection), whose per-coordinate recursion runs in
// the kernel, or full-Kalman gains computed beforehand.  With T = (I + N)^-1
// and AT = ((Q G^T) o Gam o lower) T the whole chunk is five tensor-core
// products with M = 128 rows, accumulators in TMEM:
//
//   D1 = [K; Q] G^T        (K G^T and Q G^T)          N = 64,  K = d_k
//   D2 = [K; Q] S0         (K S0 and Q S0)            N = d_v, K = d_k
//   DT = [T; Attn] T       (rows 64..127: AT)         N = 64,  K = 64
//   D3 = [T; AT] R         (E and the intra-chunk O)  N = d_v, K = 64
//   D4 = G^T Et            (S_C - A_C S0)             N = d_v, K = 64
//
// K, Q and V enter exactly (bf16); every fp32 operand (S0, G, T, AT, R, the
// scaled E) is split into two bf16 terms hi + lo and its products take two or
// three MMAs, which keeps about 16 significand bits.  T comes from a blocked
// triangular inversion on the CUDA cores.  The fp32 state master lives in TMEM.
#include <cuda.h>

#include <mutex>

#include "chunk.h"
#include "common.cuh"
#include "kernels.h"
#include "chunk_common.cuh"
#include "sm100.cuh"

namespace kdn {

namespace {

using chunk::kC;
using chunk::kWaitCycles;
using chunk::load8_bf16;
using chunk::named_arrive;
using chunk::named_sync;
using chunk::oct_sum;
using chunk::store8_split;
constexpr int kThreads = 512;   // 16 warps: warp w reads TMEM lanes 32*(w%4).., column quarter w/4
// One thread issues every tcgen05.mma and commit (a commit tracks only its own thread's products): the
// first lane of the last warp, which has no part in the diagonal-variance recursion at a chunk's start.
constexpr int kIssuer = kThreads - 32;

enum Var : int { kDelta = 0, kDiag = 1, kFull = 2 };

template <int D, int VAR>
struct Layout {
  static constexpr int NP = D / 64;                 // 64-wide panels across d
  static constexpr int KQ_PANEL = 128 * 128;        // [K; Q]: rows 0..63 K, 64..127 Q
  static constexpr int V_PANEL = 64 * 128;
  static constexpr int G_PANEL = 64 * 128;
  static constexpr int S_PANEL = D * 128;           // d_k rows
  static constexpr int RE_PANEL = 64 * 128;
  static constexpr int TAT_BYTES = 128 * 128;       // one panel of 128 rows x 64
  static constexpr int KQ_BUFS = (VAR == kDelta) ? 2 : 1;  // the delta rule reads K until the last MMA

  static constexpr int OFF_KQ = 0;
  static constexpr int KQ_BYTES = NP * KQ_PANEL;
  static constexpr int OFF_V = OFF_KQ + KQ_BUFS * KQ_BYTES;
  static constexpr int OFF_GHI = OFF_V + NP * V_PANEL;
  static constexpr int G_BYTES = (VAR == kDelta) ? 0 : NP * G_PANEL;
  static constexpr int OFF_GLO = OFF_GHI + G_BYTES;
  static constexpr int OFF_SHI = OFF_GLO + G_BYTES;
  static constexpr int OFF_SLO = OFF_SHI + NP * S_PANEL;
  static constexpr int OFF_THI = OFF_SLO + NP * S_PANEL;
  static constexpr int OFF_TLO = OFF_THI + TAT_BYTES;
  static constexpr int OFF_RHI = OFF_TLO + TAT_BYTES;
  static constexpr int OFF_RLO = OFF_RHI + NP * RE_PANEL;
  static constexpr int END = OFF_RLO + NP * RE_PANEL;
  // fp32 [64][68] scratch for N and T: inside the state panels (dead between the
  // [K;Q] S0 product and the state write-back) when they are large enough
  static constexpr int SCR_LD = 68;
  static constexpr int SCR_BYTES = 64 * SCR_LD * 4;
  static constexpr bool SCR_IN_S = NP * S_PANEL >= SCR_BYTES;
  static constexpr int OFF_NF = SCR_IN_S ? OFF_SLO : END;
  static constexpr int OFF_TF = SCR_IN_S ? OFF_SHI : END + SCR_BYTES;
  static constexpr int TOTAL = END + (SCR_IN_S ? 0 : 2 * SCR_BYTES);
  static constexpr int SMEM = TOTAL + 1024;         // + alignment slack
  // fp32 [64][D] gain scratch in the R/E area (2 * NP * 8 KB = 256 * D bytes)
  static constexpr int OFF_GF = OFF_RHI;
  // TMEM columns; T_SM holds the fp32 state master, which D4 = G^T Et accumulates onto
  static constexpr uint32_t T_D1 = 0, T_D2 = 64, T_DT = 64 + D, T_D3 = 128 + D, T_SM = 128 + 2 * D;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(128 + 3 * D <= 512, "TMEM budget");
  static_assert(TOTAL <= 224 * 1024, "shared memory budget");
};





struct Params {
  const float* beta;
  const float* a;
  const float* r;
  const float* qn;
  float qn_scalar;
  const float* gains;  // full Kalman: [BH, L, D] fp32
  float* S;
  float* p;            // diag: [BH, D]
  void* o;
  float* m;
  int out_dtype;
  int L;
  unsigned* status;
};

// Position of coordinate i within a row of the fp32 gain scratch. Within each 64-wide block the
// 4-float quads are permuted, (i % 64) = 8 p + 4 h + e  ->  32 h + 4 (p ^ 4 h) + e, so that a warp
// writing 32 consecutive coordinates, and eight lanes reading the quads h of chunks p = 0..7, each
// touch 32 distinct banks.
__device__ __forceinline__ int gf_pos(int i) {
  const int h = (i >> 2) & 1;
  return (i & ~63) | (h << 5) | ((((i >> 3) & 7) ^ (h << 2)) << 2) | (i & 3);
}

template <int D, int VAR>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_scan_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, Params P) {
  using Lay = Layout<D, VAR>;
  constexpr int NP = Lay::NP;
  constexpr int QC = D / 4;    // d_v columns per column quarter
  constexpr int LD = Lay::SCR_LD;
  constexpr int GD = D / 8;    // coordinates per thread in the per-token reductions (8 threads per token)

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Vs = sm + Lay::OFF_V;
  uint8_t* Ghi = sm + Lay::OFF_GHI;
  uint8_t* Glo = sm + Lay::OFF_GLO;
  uint8_t* Shi = sm + Lay::OFF_SHI;
  uint8_t* Slo = sm + Lay::OFF_SLO;
  uint8_t* Thi = sm + Lay::OFF_THI;
  uint8_t* Tlo = sm + Lay::OFF_TLO;
  uint8_t* Rhi = sm + Lay::OFF_RHI;
  uint8_t* Rlo = sm + Lay::OFF_RLO;
  float* Nf = reinterpret_cast<float*>(sm + Lay::OFF_NF);
  float* Tf = reinterpret_cast<float*>(sm + Lay::OFF_TF);
  float* Gf = reinterpret_cast<float*>(sm + Lay::OFF_GF);

  __shared__ float sA[2][kC], sB[2][kC], sQ[2][kC];  // a, beta|r, Qn of this chunk and the next
  __shared__ float ell[kC], Aex[kC], Arat[kC], gn[kC], en[4][kC];
  __shared__ uint64_t bar_kq[2], bar_v, bar_mma;
  __shared__ uint32_t tmem_base;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int qw = warp & 3, cq = warp >> 2;  // TMEM lane quarter, column quarter
  const int row = 32 * qw + lane;           // TMEM lane of this thread
  const int bh = blockIdx.x;
  const int L = P.L;
  const int nchunks = (L + kC - 1) / kC;

  // per-token scalars of chunk cc: read into registers early, stored into shared memory late,
  // so that the global-load latency hides behind a whole chunk
  float ra = 1.f, rb = 0.f, rq = 0.f;
  auto fetch_scalars = [&](int cc) {
    if (tid < kC) {
      const int tok = cc * kC + tid;
      const bool valid = tok < L;
      const size_t ti = (size_t)bh * L + tok;
      ra = valid ? (P.a ? P.a[ti] : 1.f) : 1.f;
      if (VAR == kDelta) rb = valid ? P.beta[ti] : 0.f;
      else rb = valid ? P.r[ti] : 1.f;
      rq = valid ? (P.qn ? P.qn[ti] : P.qn_scalar) : 0.f;
    }
  };
  auto store_scalars = [&](int buf) {
    if (tid < kC) sA[buf][tid] = ra, sB[buf][tid] = rb, sQ[buf][tid] = rq;
  };
  auto issue_kq = [&](int cc, int buf) {
    uint8_t* dst = sm + Lay::OFF_KQ + buf * Lay::KQ_BYTES;
    sm100::mbar_arrive_expect_tx(&bar_kq[buf], 2 * NP * 64 * 128);
#pragma unroll
    for (int pn = 0; pn < NP; ++pn) {
      sm100::tma_load_3d(dst + pn * Lay::KQ_PANEL, &tm_k, &bar_kq[buf], 64 * pn, cc * kC, bh);
      sm100::tma_load_3d(dst + pn * Lay::KQ_PANEL + 64 * 128, &tm_q, &bar_kq[buf], 64 * pn, cc * kC, bh);
    }
  };
  auto issue_v = [&](int cc) {
    sm100::mbar_arrive_expect_tx(&bar_v, NP * 64 * 128);
#pragma unroll
    for (int pn = 0; pn < NP; ++pn) sm100::tma_load_3d(Vs + pn * Lay::V_PANEL, &tm_v, &bar_v, 64 * pn, cc * kC, bh);
  };

  if (tid == 0) {
    sm100::prefetch_tmap(&tm_q);
    sm100::prefetch_tmap(&tm_k);
    sm100::prefetch_tmap(&tm_v);
    sm100::mbar_init(&bar_kq[0], 1);
    sm100::mbar_init(&bar_kq[1], 1);
    sm100::mbar_init(&bar_v, 1);
    sm100::mbar_init(&bar_mma, 1);
    sm100::fence_mbar_init();
    issue_kq(0, 0);  // chunk c issues chunk c + 1
    issue_v(0);
  }
  if (warp == 0) {
    sm100::tmem_alloc(&tmem_base, Lay::TMEM_COLS);
    sm100::tmem_relinquish();
  }
  fetch_scalars(0);
  store_scalars(0);
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = tmem_base;
  const uint32_t t_lane = static_cast<uint32_t>(32 * qw) << 16;

  // ---- state: thread (lane row, column quarter) owns S[row][cq*QC .. +QC); fp32 master in TMEM,
  //      bf16 hi/lo panels in shared memory for the [K;Q] S0 product
  const bool s_owner = row < D;
  float* Sg = P.S + (size_t)bh * D * D;
  auto write_state_panels = [&](const float (&x)[QC]) {
#pragma unroll
    for (int u = 0; u < QC / 8; ++u) {
      const int c = cq * QC + 8 * u;  // d_v column
      float y[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) y[e] = x[8 * u + e];
      store8_split(Shi, Slo, (c / 64) * Lay::S_PANEL + sm100::sw128_chunk(row, (c % 64) / 8), y);
    }
  };
  if (s_owner) {  // warp-uniform: D is 64 or 128
    float x[QC];
#pragma unroll
    for (int c = 0; c < QC; c += 4) {
      const float4 v4 = *reinterpret_cast<const float4*>(Sg + (size_t)row * D + cq * QC + c);
      x[c] = v4.x, x[c + 1] = v4.y, x[c + 2] = v4.z, x[c + 3] = v4.w;
    }
    sm100::tmem_st<QC>(tmem + t_lane + Lay::T_SM + cq * QC, x);
    write_state_panels(x);
    sm100::tmem_wait_st();
  }
  // diagonal covariance: coordinate tid (threads 0 .. D-1)
  float pcur = 1.f;
  if (VAR == kDiag && tid < D) pcur = P.p[(size_t)bh * D + tid];
  sm100::fence_async_smem();
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();

  uint32_t mma_phase = 0;
  bool aborted = false;
  // one thread waits on the mbarriers, then a CTA-wide vote
  auto wait_all = [&](uint64_t* b1, uint32_t par1, uint64_t* b2, uint32_t par2) -> bool {
    int bad = 0;
    if (tid == 0) {
      bad = !sm100::mbar_wait_bounded(b1, par1, kWaitCycles);
      if (!bad && b2 != nullptr) bad = !sm100::mbar_wait_bounded(b2, par2, kWaitCycles);
    }
    bad = __syncthreads_or(bad);
    if (bad && tid == 0) raise_status(P.status, kStatusTimeout);
    sm100::tc_fence_after();
    return !bad;
  };

  const uint32_t shi = sm100::smem_u32(Shi), slo = sm100::smem_u32(Slo);
  const uint32_t ghi = sm100::smem_u32(Ghi), glo = sm100::smem_u32(Glo);
  const uint32_t thi = sm100::smem_u32(Thi), tlo = sm100::smem_u32(Tlo);
  const uint32_t rhi = sm100::smem_u32(Rhi), rlo = sm100::smem_u32(Rlo);

  for (int c = 0; c < nchunks; ++c) {
    const int t0 = c * kC;
    const int kb = (Lay::KQ_BUFS == 2) ? (c & 1) : 0;
    const int sb = c & 1;
    uint8_t* KQ = sm + Lay::OFF_KQ + kb * Lay::KQ_BYTES;
    const uint32_t kq0 = sm100::smem_u32(KQ);
    const float* a_c = sA[sb];
    const float* b_c = sB[sb];
    const float* q_c = sQ[sb];

    // ---------------------------------------------------------------- K, Q of this chunk; start [K;Q] S0
    if (!wait_all(&bar_kq[kb], (Lay::KQ_BUFS == 2) ? ((c >> 1) & 1) : (c & 1), nullptr, 0)) { aborted = true; break; }
    if (tid == 0 && Lay::KQ_BUFS == 2 && c + 1 < nchunks) issue_kq(c + 1, kb ^ 1);
    if (tid == kIssuer) {
      constexpr uint32_t id1 = sm100::idesc_bf16(128, 64, false, false);
      constexpr uint32_t id2 = sm100::idesc_bf16(128, D, false, true);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t koff = (ks / 4) * Lay::KQ_PANEL + (ks % 4) * 32;
        const uint64_t a = sm100::smem_desc(kq0 + koff, 16, 1024);
        sm100::mma_bf16(tmem + Lay::T_D2, a, sm100::smem_desc(shi + ks * 2048, Lay::S_PANEL, 1024), id2, ks > 0);
        sm100::mma_bf16(tmem + Lay::T_D2, a, sm100::smem_desc(slo + ks * 2048, Lay::S_PANEL, 1024), id2, true);
        if (VAR == kDelta)  // G = K: [K;Q] K^T now
          sm100::mma_bf16(tmem + Lay::T_D1, a, sm100::smem_desc(kq0 + koff, 16, 1024), id1, ks > 0);
      }
      if (VAR == kDelta) sm100::mma_commit(&bar_mma);
    }
    if (c + 1 < nchunks) fetch_scalars(c + 1);

    // ---------------------------------------------------------------- gates
    if (warp == 1) {
      // inclusive prefix sums of log a over the chunk (a gate of 0 enters as exp(-60))
      float x0 = a_c[lane], x1 = a_c[32 + lane];
      x0 = x0 > 0.f ? fmaxf(__logf(x0), -60.f) : -60.f;
      x1 = x1 > 0.f ? fmaxf(__logf(x1), -60.f) : -60.f;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y0 = __shfl_up_sync(0xffffffffu, x0, o), y1 = __shfl_up_sync(0xffffffffu, x1, o);
        if (lane >= o) x0 += y0, x1 += y1;
      }
      x1 += __shfl_sync(0xffffffffu, x0, 31);
      const float lC = __shfl_sync(0xffffffffu, x1, 31);
      ell[lane] = x0, ell[32 + lane] = x1;
      Aex[lane] = __expf(x0), Aex[32 + lane] = __expf(x1);
      Arat[lane] = __expf(lC - x0), Arat[32 + lane] = __expf(lC - x1);  // A_C / A_i without a division
    }
    // ---------------------------------------------------------------- diagonal variances
    if (VAR == kDiag && tid < D) {
      // Per coordinate i (independent of v and S): p^- = a^2 p + Qn, pk = p^- k, p <- p^- r / (r + pk k).
      // The step is a linear-fractional map of p, so it runs on the homogeneous pair p = x / y:
      //   x^- = a^2 x + Qn y,  x <- r x^-,  y <- r y + k^2 x^-,
      // which keeps the division out of the serial chain (three multiply-adds per token); pk = x^- k / y
      // hangs off it. Every four tokens the pair is rescaled by a power of two, so y stays in [1, 2).
      const uint8_t* Kp = KQ + (tid / 64) * Lay::KQ_PANEL;
      const int gpos = gf_pos(tid);
      float x = pcur, y = 1.f;
#pragma unroll 1
      for (int t8 = 0; t8 < kC; t8 += 8) {
        float kk[8], aa[8], rr8[8], qq[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          kk[u] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(Kp + sm100::sw128(t8 + u, tid % 64)));
          aa[u] = a_c[t8 + u], rr8[u] = b_c[t8 + u], qq[u] = q_c[t8 + u];
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float xm = fmaf(aa[u] * aa[u], x, qq[u] * y);
          Gf[(t8 + u) * D + gpos] = __fdividef(xm * kk[u], y);
          x = rr8[u] * xm;
          y = fmaf(kk[u] * kk[u], xm, rr8[u] * y);
          if (u % 4 == 3) {
            const int ey = min((__float_as_int(y) >> 23) & 0xff, 253);
            const float sc = __int_as_float((254 - ey) << 23);  // 2^(127 - ey), exact
            x *= sc, y *= sc;
          }
        }
      }
      pcur = __fdividef(x, y);
    }
    __syncthreads();

    // ---------------------------------------------------------------- gains: norms, hi/lo panels (8 threads per token)
    {
      // Thread `part` of token t takes the 16-byte chunk `part` of every 64-wide panel: coordinates
      // 64 pn + 8 part .. + 7, so each group of eight lanes reads and writes one whole 128-byte row.
      const int t = tid >> 3, part = tid & 7;
      float kv[GD];
#pragma unroll
      for (int pn = 0; pn < NP; ++pn) {
        float x[8];
        load8_bf16(KQ + pn * Lay::KQ_PANEL, sm100::sw128_chunk(t, part), x);
#pragma unroll
        for (int e = 0; e < 8; ++e) kv[8 * pn + e] = x[e];
      }
      if (VAR == kDelta) {
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < GD; ++e) s = fmaf(kv[e], kv[e], s);
        s = oct_sum(s);
        if (part == 0) gn[t] = b_c[t] * b_c[t] * s;
      } else {
        float g[GD];
        if (VAR == kDiag) {
#pragma unroll
          for (int pn = 0; pn < NP; ++pn)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float4 x = *reinterpret_cast<const float4*>(Gf + t * D + gf_pos(64 * pn + 8 * part + 4 * h));
              g[8 * pn + 4 * h] = x.x, g[8 * pn + 4 * h + 1] = x.y, g[8 * pn + 4 * h + 2] = x.z, g[8 * pn + 4 * h + 3] = x.w;
            }
          float s = 0.f;
#pragma unroll
          for (int e = 0; e < GD; ++e) s = fmaf(g[e], kv[e], s);
          s = oct_sum(s) + b_c[t];
          if (part == 0 && !(s > 0.f && isfinite(s))) raise_status(P.status, kStatusNumeric);
          const float inv_s = 1.f / s;
#pragma unroll
          for (int e = 0; e < GD; ++e) g[e] *= inv_s;
        } else {
          const bool valid = t0 + t < L;
          const float* gp = P.gains + ((size_t)bh * L + t0 + t) * D + 8 * part;
#pragma unroll
          for (int pn = 0; pn < NP; ++pn)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
              if (valid) x = *reinterpret_cast<const float4*>(gp + 64 * pn + 4 * h);
              g[8 * pn + 4 * h] = x.x, g[8 * pn + 4 * h + 1] = x.y, g[8 * pn + 4 * h + 2] = x.z, g[8 * pn + 4 * h + 3] = x.w;
            }
        }
        float n2 = 0.f;
#pragma unroll
        for (int e = 0; e < GD; ++e) n2 = fmaf(g[e], g[e], n2);
        n2 = oct_sum(n2);
        if (part == 0) gn[t] = n2;
#pragma unroll
        for (int pn = 0; pn < NP; ++pn) {
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = g[8 * pn + e];
          store8_split(Ghi, Glo, pn * Lay::G_PANEL + sm100::sw128_chunk(t, part), x);
        }
      }
    }
    sm100::fence_async_smem();
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();

    // ---------------------------------------------------------------- D1 = [K;Q] G^T (Kalman gains)
    if (tid == kIssuer && VAR != kDelta) {
      constexpr uint32_t id1 = sm100::idesc_bf16(128, 64, false, false);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t koff = (ks / 4) * Lay::KQ_PANEL + (ks % 4) * 32;
        const uint32_t goff = (ks / 4) * Lay::G_PANEL + (ks % 4) * 32;
        const uint64_t a = sm100::smem_desc(kq0 + koff, 16, 1024);
        sm100::mma_bf16(tmem + Lay::T_D1, a, sm100::smem_desc(ghi + goff, 16, 1024), id1, ks > 0);
        sm100::mma_bf16(tmem + Lay::T_D1, a, sm100::smem_desc(glo + goff, 16, 1024), id1, true);
      }
      sm100::mma_commit(&bar_mma);
    }
    if (!wait_all(&bar_mma, mma_phase, &bar_v, c & 1)) { aborted = true; break; }
    mma_phase ^= 1;
    if (tid == 0 && Lay::KQ_BUFS == 1 && c + 1 < nchunks) issue_kq(c + 1, 0);  // K, Q of this chunk are dead

    // ---------------------------------------------------------------- N, R (lanes 0..63) | Attn, T (lanes 64..127)
    // The warps that own TMEM lanes 0..63 ([K;Q] rows of K) build N, hand it over through a named
    // barrier and then build R; the warps that own lanes 64..127 build Attn and then invert I + N.
    if (qw < 2) {
      const int i = row;  // token in chunk
      {
        // N_ij = (K G^T)_ij Gam_ij for j < i, columns 16 cq .. 16 cq + 15
        float Y[16];
        sm100::tmem_ld16(tmem + t_lane + Lay::T_D1 + 16 * cq, Y);
        sm100::tmem_wait_ld();
        const float li = ell[i];
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          float v4[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int j = 16 * cq + e + u;
            v4[u] = (j < i) ? Y[e + u] * __expf(li - ell[j]) * (VAR == kDelta ? b_c[j] : 1.f) : 0.f;
          }
          *reinterpret_cast<float4*>(Nf + i * LD + 16 * cq + e) = make_float4(v4[0], v4[1], v4[2], v4[3]);
        }
      }
      named_arrive(1, kThreads);  // N is ready
      const float Ai = Aex[i];
      float X[QC];
      sm100::tmem_ld<QC>(tmem + t_lane + Lay::T_D2 + cq * QC, X);
      sm100::tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < QC / 8; ++u) {
        const int cb = cq * QC + 8 * u;
        const uint32_t off = (cb / 64) * Lay::V_PANEL + sm100::sw128_chunk(i, (cb % 64) / 8);
        float vv[8], x[8];
        load8_bf16(Vs, off, vv);
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = fmaf(-Ai, X[8 * u + e], vv[e]);
        store8_split(Rhi, Rlo, off, x);
      }
    } else {
      const int gt = (qw - 2) * 32 + lane + 64 * cq;  // 0..255 within this group
      {
        // Attn_ij = (Q G^T)_ij Gam_ij for j <= i, into rows 64.. of the [T; AT] panel
        const int i = row - 64;
        float Y[16];
        sm100::tmem_ld16(tmem + t_lane + Lay::T_D1 + 16 * cq, Y);
        sm100::tmem_wait_ld();
        const float li = ell[i];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int j = 16 * cq + 8 * h + e;
            x[e] = (j <= i) ? Y[8 * h + e] * __expf(li - ell[j]) * (VAR == kDelta ? b_c[j] : 1.f) : 0.f;
          }
          store8_split(Thi, Tlo, sm100::sw128_chunk(64 + i, 2 * cq + h), x);
        }
      }
      named_sync(1, kThreads);  // wait for N
      // ---- T = (I + N)^-1 (group of the 256 threads that own lanes 64..127)
      chunk::invert_unit_lower_64(Nf, Tf, gt, [] { named_sync(2, kThreads / 2); });
      // T (unit diagonal, zero above) as bf16 hi/lo into rows 0..63 of the [T; AT] panel
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int e = gt + 256 * h;
        const int i = e >> 3, c8 = e & 7;
        const float4 lo4 = *reinterpret_cast<const float4*>(Tf + i * LD + 8 * c8);
        const float4 hi4 = *reinterpret_cast<const float4*>(Tf + i * LD + 8 * c8 + 4);
        const float tv[8] = {lo4.x, lo4.y, lo4.z, lo4.w, hi4.x, hi4.y, hi4.z, hi4.w};
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int j = 8 * c8 + u;
          x[u] = (j < i) ? tv[u] : (j == i ? 1.f : 0.f);
        }
        store8_split(Thi, Tlo, sm100::sw128_chunk(i, c8), x);
      }
    }
    sm100::fence_async_smem();
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    if (tid == 0 && c + 1 < nchunks) issue_v(c + 1);  // V of this chunk is dead

    // ---------------------------------------------------------------- DT = [T; Attn] T  (rows 64..127: AT)
    if (tid == kIssuer) {
      constexpr uint32_t id = sm100::idesc_bf16(128, 64, false, true);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t ah = sm100::smem_desc(thi + ks * 32, 16, 1024), al = sm100::smem_desc(tlo + ks * 32, 16, 1024);
        const uint64_t bh_ = sm100::smem_desc(thi + ks * 2048, 16, 1024), bl = sm100::smem_desc(tlo + ks * 2048, 16, 1024);
        sm100::mma_bf16(tmem + Lay::T_DT, ah, bh_, id, ks > 0);
        sm100::mma_bf16(tmem + Lay::T_DT, al, bh_, id, true);
        sm100::mma_bf16(tmem + Lay::T_DT, ah, bl, id, true);
      }
      sm100::mma_commit(&bar_mma);
    }
    if (!wait_all(&bar_mma, mma_phase, nullptr, 0)) { aborted = true; break; }
    mma_phase ^= 1;
    if (qw >= 2) {
      const int i = row - 64;
      float X[16];
      sm100::tmem_ld16(tmem + t_lane + Lay::T_DT + 16 * cq, X);
      sm100::tmem_wait_ld();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = X[8 * h + e];
        store8_split(Thi, Tlo, sm100::sw128_chunk(64 + i, 2 * cq + h), x);
      }
    }
    sm100::fence_async_smem();
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();

    // ---------------------------------------------------------------- D3 = [T; AT] R
    if (tid == kIssuer) {
      constexpr uint32_t id = sm100::idesc_bf16(128, D, false, true);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t ah = sm100::smem_desc(thi + ks * 32, 16, 1024), al = sm100::smem_desc(tlo + ks * 32, 16, 1024);
        const uint64_t bh_ = sm100::smem_desc(rhi + ks * 2048, Lay::RE_PANEL, 1024);
        const uint64_t bl = sm100::smem_desc(rlo + ks * 2048, Lay::RE_PANEL, 1024);
        sm100::mma_bf16(tmem + Lay::T_D3, ah, bh_, id, ks > 0);
        sm100::mma_bf16(tmem + Lay::T_D3, al, bh_, id, true);
        sm100::mma_bf16(tmem + Lay::T_D3, ah, bl, id, true);
      }
      sm100::mma_commit(&bar_mma);
    }
    if (!wait_all(&bar_mma, mma_phase, nullptr, 0)) { aborted = true; break; }
    mma_phase ^= 1;

    // ---------------------------------------------------------------- E -> scaled E panels; O out; S master *= A_C
    const float AC = Aex[kC - 1];
    if (qw < 2) {
      const int i = row;
      const float sc = Arat[i] * (VAR == kDelta ? b_c[i] : 1.f);
      float X[QC];
      sm100::tmem_ld<QC>(tmem + t_lane + Lay::T_D3 + cq * QC, X);
      sm100::tmem_wait_ld();
      float es = 0.f;
#pragma unroll
      for (int u = 0; u < QC / 8; ++u) {
        const int cb = cq * QC + 8 * u;
        float x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          es = fmaf(X[8 * u + e], X[8 * u + e], es);
          x[e] = X[8 * u + e] * sc;
        }
        store8_split(Rhi, Rlo, (cb / 64) * Lay::RE_PANEL + sm100::sw128_chunk(i, (cb % 64) / 8), x);
      }
      en[cq][i] = es;
    } else {
      const int i = row - 64;
      const int tok = t0 + i;
      const float Ai = Aex[i];
      float Y[QC], Oi[QC];
      sm100::tmem_ld<QC>(tmem + t_lane + Lay::T_D2 + cq * QC, Y);
      sm100::tmem_ld<QC>(tmem + t_lane + Lay::T_D3 + cq * QC, Oi);
      sm100::tmem_wait_ld();
      if (tok < L) {
        const size_t off = ((size_t)bh * L + tok) * D + cq * QC;
        if (P.out_dtype == kF32) {
          float* op = reinterpret_cast<float*>(P.o) + off;
#pragma unroll
          for (int e = 0; e < QC; e += 4)
            *reinterpret_cast<float4*>(op + e) = make_float4(fmaf(Ai, Y[e], Oi[e]), fmaf(Ai, Y[e + 1], Oi[e + 1]),
                                                             fmaf(Ai, Y[e + 2], Oi[e + 2]), fmaf(Ai, Y[e + 3], Oi[e + 3]));
        } else {
          __nv_bfloat16* op = reinterpret_cast<__nv_bfloat16*>(P.o) + off;
#pragma unroll
          for (int e = 0; e < QC; e += 8) {
            __align__(16) __nv_bfloat16 h[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) h[u] = __float2bfloat16_rn(fmaf(Ai, Y[e + u], Oi[e + u]));
            *reinterpret_cast<uint4*>(op + e) = *reinterpret_cast<const uint4*>(h);
          }
        }
      }
    }
    if (s_owner) {  // the product Gm^T Et accumulates onto A_C S0
      float x[QC];
      sm100::tmem_ld<QC>(tmem + t_lane + Lay::T_SM + cq * QC, x);
      sm100::tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < QC; ++e) x[e] *= AC;
      sm100::tmem_st<QC>(tmem + t_lane + Lay::T_SM + cq * QC, x);
      sm100::tmem_wait_st();
    }
    sm100::fence_async_smem();
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();

    // ---------------------------------------------------------------- S master += G^T Et
    if (tid == kIssuer) {
      constexpr uint32_t id = sm100::idesc_bf16(128, D, true, true);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t bh_ = sm100::smem_desc(rhi + ks * 2048, Lay::RE_PANEL, 1024);
        const uint64_t bl = sm100::smem_desc(rlo + ks * 2048, Lay::RE_PANEL, 1024);
        if (VAR == kDelta) {
          const uint64_t ak = sm100::smem_desc(kq0 + ks * 2048, Lay::KQ_PANEL, 1024);
          sm100::mma_bf16(tmem + Lay::T_SM, ak, bh_, id, true);
          sm100::mma_bf16(tmem + Lay::T_SM, ak, bl, id, true);
        } else {
          const uint64_t ah = sm100::smem_desc(ghi + ks * 2048, Lay::G_PANEL, 1024);
          const uint64_t al = sm100::smem_desc(glo + ks * 2048, Lay::G_PANEL, 1024);
          sm100::mma_bf16(tmem + Lay::T_SM, ah, bh_, id, true);
          sm100::mma_bf16(tmem + Lay::T_SM, al, bh_, id, true);
          sm100::mma_bf16(tmem + Lay::T_SM, ah, bl, id, true);
        }
      }
      sm100::mma_commit(&bar_mma);
    }
    if (tid < kC && P.m != nullptr && t0 + tid < L)
      P.m[(size_t)bh * L + t0 + tid] = sqrtf(gn[tid]) * sqrtf(en[0][tid] + en[1][tid] + en[2][tid] + en[3][tid]);
    if (!wait_all(&bar_mma, mma_phase, nullptr, 0)) { aborted = true; break; }
    mma_phase ^= 1;

    // ---------------------------------------------------------------- state panels for the next chunk
    if (s_owner) {
      float x[QC];
      sm100::tmem_ld<QC>(tmem + t_lane + Lay::T_SM + cq * QC, x);
      sm100::tmem_wait_ld();
      write_state_panels(x);
    }
    if (c + 1 < nchunks) store_scalars(sb ^ 1);
    sm100::fence_async_smem();
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
  }

  // ---- write back the state (and the diagonal covariance)
  if (!aborted) {
    if (s_owner) {
      float x[QC];
      sm100::tmem_ld<QC>(tmem + t_lane + Lay::T_SM + cq * QC, x);
      sm100::tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < QC; e += 4)
        *reinterpret_cast<float4*>(Sg + (size_t)row * D + cq * QC + e) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
    }
    if (VAR == kDiag && tid < D) P.p[(size_t)bh * D + tid] = pcur;
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 0) sm100::tmem_dealloc(tmem, Lay::TMEM_COLS);
}

// ------------------------------------------------------------------------------------------- host side

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

template <int D, int VAR>
cudaError_t launch_typed(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const Params& p, int BH,
                         cudaStream_t stream) {
  using Lay = Layout<D, VAR>;
  cudaError_t e = cudaFuncSetAttribute(chunk_scan_kernel<D, VAR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Lay::SMEM);
  if (e != cudaSuccess) return e;
  chunk_scan_kernel<D, VAR><<<BH, kThreads, Lay::SMEM, stream>>>(q, k, v, p);
  return cudaGetLastError();
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
  *kernel = variant == KDN_KALMAN_FULL ? "kalman_pside_kernel"
                                       : (d.dk == 128 ? "chunk_scan_ws_kernel" : "chunk_scan_kernel");
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
  if (d.dk == 128) return launch_chunk_ws(variant, d, a, gains, stream);
  const int BH = a.BH;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_impl(&tq, a.q, BH, a.L, d.dk) || !make_tmap_impl(&tk, a.k, BH, a.L, d.dk) ||
      !make_tmap_impl(&tv, a.v, BH, a.L, d.dv))
    return cudaErrorInvalidValue;
  Params p{};
  p.beta = a.beta, p.a = a.a, p.r = a.r, p.qn = a.qn, p.qn_scalar = a.qn_scalar;
  p.S = a.S, p.o = a.o, p.m = a.m, p.out_dtype = a.out_dtype, p.L = a.L, p.status = a.status;
  if (variant == KDN_KALMAN_FULL) {
    if (gains == nullptr) return cudaErrorInvalidValue;
    p.gains = gains;
    return launch_typed<64, kFull>(tq, tk, tv, p, BH, stream);
  }
  if (variant == KDN_KALMAN_DIAG) {
    p.p = a.P;
    return launch_typed<64, kDiag>(tq, tk, tv, p, BH, stream);
  }
  return launch_typed<64, kDelta>(tq, tk, tv, p, BH, stream);
}

}  // namespace kdn
