// Chunked scan on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
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
// triangular inversion on the CUDA cores.  The state S is fp32 in registers.
#include <cuda.h>

#include <mutex>

#include "chunk.h"
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace kdn {

namespace {

constexpr int kC = 64;          // tokens per chunk
constexpr int kThreads = 256;   // 8 warps: warp w reads TMEM lanes 32*(w%4).., column half w/4
constexpr long long kWaitCycles = 2000000000LL;  // bounded waits: about one second

enum Var : int { kDelta = 0, kDiag = 1, kFull = 2 };

template <int D, int VAR>
struct Layout {
  static constexpr int NP = D / 64;                 // 64-wide panels across d
  static constexpr int KQ_PANEL = 128 * 128;        // [K; Q] rows 0..63 K, 64..127 Q
  static constexpr int V_PANEL = 64 * 128;
  static constexpr int G_PANEL = 64 * 128;
  static constexpr int S_PANEL = D * 128;           // d_k rows
  static constexpr int RE_PANEL = 64 * 128;
  static constexpr int TAT_BYTES = 128 * 128;       // one panel of 128 rows x 64

  static constexpr int OFF_KQ = 0;
  static constexpr int OFF_V = OFF_KQ + NP * KQ_PANEL;
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
  // fp32 [64][64] scratch for N and T; alias dead buffers when they are large enough
  static constexpr int NF_BYTES = 64 * 64 * 4;
  static constexpr bool NF_IN_V = NP * V_PANEL >= NF_BYTES;
  static constexpr bool TF_IN_S = NP * S_PANEL >= NF_BYTES;
  static constexpr int OFF_NF = NF_IN_V ? OFF_V : END;
  static constexpr int OFF_TF = TF_IN_S ? OFF_SHI : (NF_IN_V ? END : END + NF_BYTES);
  static constexpr int TOTAL = END + (NF_IN_V ? 0 : NF_BYTES) + (TF_IN_S ? 0 : NF_BYTES);
  static constexpr int SMEM = TOTAL + 1024;         // + alignment slack
  // fp32 [64][D] gain scratch (diag / full) in the R/E area: 2 * NP * 8 KB = 256 * D bytes
  static constexpr int OFF_GF = OFF_RHI;
  // TMEM columns
  static constexpr uint32_t T_D1 = 0, T_D2 = 64, T_DT = 64 + D, T_D3 = 128 + D, T_D4 = 128 + 2 * D;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(128 + 3 * D <= 512, "TMEM budget");
  static_assert(TOTAL <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ int fidx(int i, int j) { return i * 64 + (j ^ (i & 31)); }  // [64][64] fp32, bank-spread

__device__ __forceinline__ void store8_split(uint8_t* hi, uint8_t* lo, uint32_t off, const float (&x)[8]) {
  __align__(16) __nv_bfloat16 h[8], l[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) sm100::split_bf16(x[e], h[e], l[e]);
  *reinterpret_cast<uint4*>(hi + off) = *reinterpret_cast<const uint4*>(h);
  *reinterpret_cast<uint4*>(lo + off) = *reinterpret_cast<const uint4*>(l);
}

__device__ __forceinline__ float ld_bf16(const uint8_t* base, uint32_t off) {
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + off));
}

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

template <int D, int VAR>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_scan_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, Params P) {
  using Lay = Layout<D, VAR>;
  constexpr int NP = Lay::NP;
  constexpr int HALF = D / 2;  // columns of d_v per column half

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* KQ = sm + Lay::OFF_KQ;
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

  __shared__ float ell[kC], Aex[kC], sc1[kC], sc2[kC], sc3[kC], gn[kC], en[2][kC];
  __shared__ uint64_t bar_load, bar_mma;
  __shared__ uint32_t tmem_base;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int qw = warp & 3, ch = warp >> 2;
  const int row = 32 * qw + lane;  // TMEM lane of this thread
  const int bh = blockIdx.x;
  const int L = P.L;
  const int nchunks = (L + kC - 1) / kC;

  if (tid == 0) {
    sm100::prefetch_tmap(&tm_q);
    sm100::prefetch_tmap(&tm_k);
    sm100::prefetch_tmap(&tm_v);
    sm100::mbar_init(&bar_load, 1);
    sm100::mbar_init(&bar_mma, 1);
    sm100::fence_mbar_init();
  }
  if (warp == 0) {
    sm100::tmem_alloc(&tmem_base, Lay::TMEM_COLS);
    sm100::tmem_relinquish();
  }

  // ---- initial state: fp32 master in registers, bf16 hi/lo panels for the MMAs
  float Sr[HALF];
  const bool s_owner = row < D;
  float* Sg = P.S + (size_t)bh * D * D;
  if (s_owner) {
#pragma unroll
    for (int c = 0; c < HALF; c += 4) {
      const float4 x = *reinterpret_cast<const float4*>(Sg + (size_t)row * D + ch * HALF + c);
      Sr[c] = x.x, Sr[c + 1] = x.y, Sr[c + 2] = x.z, Sr[c + 3] = x.w;
    }
  }
  // per-coordinate diagonal covariance, owned by threads 128 + i
  float pcur = 1.f;
  const int pi = tid - 128;
  if (VAR == kDiag && pi >= 0 && pi < D) pcur = P.p[(size_t)bh * D + pi];

  auto write_state_panels = [&]() {
    if (!s_owner) return;
#pragma unroll
    for (int c8 = 0; c8 < HALF / 8; ++c8) {
      const int c = ch * HALF + c8 * 8;  // d_v column
      float x[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = Sr[c8 * 8 + e];
      store8_split(Shi, Slo, (c / 64) * Lay::S_PANEL + sm100::sw128_chunk(row, (c % 64) / 8), x);
    }
  };
  write_state_panels();
  sm100::fence_async_smem();
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = tmem_base;
  const uint32_t t_lane = static_cast<uint32_t>(32 * qw) << 16;

  uint32_t mma_phase = 0;
  bool aborted = false;
  // single-thread wait on an mbarrier, then a CTA-wide vote
  auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
    int bad = 0;
    if (tid == 0) bad = !sm100::mbar_wait_bounded(bar, parity, kWaitCycles);
    bad = __syncthreads_or(bad);
    if (bad && tid == 0) raise_status(P.status, kStatusTimeout);
    sm100::tc_fence_after();
    return !bad;
  };

  const uint32_t kq0 = sm100::smem_u32(KQ);

  for (int c = 0; c < nchunks && !aborted; ++c) {
    const int t0 = c * kC;
    // ---------------------------------------------------------------- stage inputs
    if (tid == 0) {
      sm100::mbar_arrive_expect_tx(&bar_load, 3 * NP * 64 * 128);
#pragma unroll
      for (int pn = 0; pn < NP; ++pn) {
        sm100::tma_load_3d(KQ + pn * Lay::KQ_PANEL, &tm_k, &bar_load, 64 * pn, t0, bh);
        sm100::tma_load_3d(KQ + pn * Lay::KQ_PANEL + 64 * 128, &tm_q, &bar_load, 64 * pn, t0, bh);
        sm100::tma_load_3d(Vs + pn * Lay::V_PANEL, &tm_v, &bar_load, 64 * pn, t0, bh);
      }
    }
    if (tid < kC) {
      const int tok = t0 + tid;
      const bool valid = tok < L;
      const size_t ti = (size_t)bh * L + tok;
      sc1[tid] = valid ? (P.a ? P.a[ti] : 1.f) : 1.f;                          // a
      if (VAR == kDelta) sc2[tid] = valid ? P.beta[ti] : 0.f;                  // beta
      else sc2[tid] = valid ? P.r[ti] : 1.f;                                   // r
      sc3[tid] = valid ? (P.qn ? P.qn[ti] : P.qn_scalar) : 0.f;                // Qn
    }
    if (!wait_all(&bar_load, c & 1)) { aborted = true; break; }

    // ---------------------------------------------------------------- gates and gains
    if (warp == 0) {
      // inclusive prefix sums of log a over the chunk (a gate of 0 enters as exp(-60))
      float x0 = sc1[lane], x1 = sc1[32 + lane];
      x0 = x0 > 0.f ? fmaxf(__logf(x0), -60.f) : -60.f;
      x1 = x1 > 0.f ? fmaxf(__logf(x1), -60.f) : -60.f;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y0 = __shfl_up_sync(0xffffffffu, x0, o), y1 = __shfl_up_sync(0xffffffffu, x1, o);
        if (lane >= o) x0 += y0, x1 += y1;
      }
      x1 += __shfl_sync(0xffffffffu, x0, 31);
      ell[lane] = x0, ell[32 + lane] = x1;
      Aex[lane] = expf(x0), Aex[32 + lane] = expf(x1);
    }
    if (VAR == kDiag && pi >= 0 && pi < D) {
      // per-coordinate variance recursion (independent of v and S):
      // p^- = a^2 p + Qn, pk = p^- k, p <- p^- r / (r + p^- k^2)
      const uint8_t* Kp = KQ + (pi / 64) * Lay::KQ_PANEL;
      for (int t = 0; t < kC; ++t) {
        const float at = sc1[t], rt = sc2[t];
        const float kt = ld_bf16(Kp, sm100::sw128(t, pi % 64));
        const float pp = fmaf(at * at, pcur, sc3[t]);
        const float pk = pp * kt;
        Gf[t * D + pi] = pk;
        pcur = pp * rt / fmaf(pk, kt, rt);
      }
    }
    if (VAR == kFull) {
      for (int idx = tid; idx < kC * D / 4; idx += kThreads) {
        const int t = idx / (D / 4), i4 = idx % (D / 4);
        float4 g = make_float4(0.f, 0.f, 0.f, 0.f);
        if (t0 + t < L) g = *reinterpret_cast<const float4*>(P.gains + ((size_t)bh * L + t0 + t) * D + 4 * i4);
        *reinterpret_cast<float4*>(Gf + t * D + 4 * i4) = g;
      }
    }
    __syncthreads();
    // gains: normalise (diag), squared norms, bf16 hi/lo panels of G
    for (int t = warp; t < kC; t += kThreads / 32) {
      if (VAR == kDelta) {
        float s = 0.f;
        for (int i = lane; i < D; i += 32) {
          const float kv = ld_bf16(KQ + (i / 64) * Lay::KQ_PANEL, sm100::sw128(t, i % 64));
          s = fmaf(kv, kv, s);
        }
        s = warp_sum(s);
        if (lane == 0) gn[t] = sc2[t] * sc2[t] * s;
      } else {
        float inv_s = 1.f;
        if (VAR == kDiag) {
          float s = 0.f;
          for (int i = lane; i < D; i += 32)
            s = fmaf(Gf[t * D + i], ld_bf16(KQ + (i / 64) * Lay::KQ_PANEL, sm100::sw128(t, i % 64)), s);
          s = warp_sum(s) + sc2[t];
          if (lane == 0 && !(s > 0.f && isfinite(s))) raise_status(P.status, kStatusNumeric);
          inv_s = 1.f / s;
        }
        float n2 = 0.f;
        for (int i = lane; i < D; i += 32) {
          const float g = Gf[t * D + i] * inv_s;
          Gf[t * D + i] = g;
          n2 = fmaf(g, g, n2);
        }
        n2 = warp_sum(n2);
        if (lane == 0) gn[t] = n2;
      }
    }
    if (VAR != kDelta) {
      __syncthreads();
      for (int idx = tid; idx < kC * D / 8; idx += kThreads) {
        const int t = idx / (D / 8), c8 = idx % (D / 8);
        float x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = Gf[t * D + 8 * c8 + e];
        store8_split(Ghi, Glo, (c8 / 8) * Lay::G_PANEL + sm100::sw128_chunk(t, c8 % 8), x);
      }
    }
    sm100::fence_async_smem();
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();

    // ---------------------------------------------------------------- D1 = [K;Q] G^T, D2 = [K;Q] S0
    if (tid == 0) {
      constexpr uint32_t id1 = sm100::idesc_bf16(128, 64, false, false);
      constexpr uint32_t id2 = sm100::idesc_bf16(128, D, false, true);
      const uint32_t ghi = sm100::smem_u32(Ghi), glo = sm100::smem_u32(Glo);
      const uint32_t shi = sm100::smem_u32(Shi), slo = sm100::smem_u32(Slo);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t koff = (ks / 4) * Lay::KQ_PANEL + (ks % 4) * 32;
        const uint64_t a = sm100::smem_desc(kq0 + koff, 16, 1024);
        if (VAR == kDelta) {
          sm100::mma_bf16(tmem + Lay::T_D1, a, sm100::smem_desc(kq0 + koff, 16, 1024), id1, ks > 0);
        } else {
          const uint32_t goff = (ks / 4) * Lay::G_PANEL + (ks % 4) * 32;
          sm100::mma_bf16(tmem + Lay::T_D1, a, sm100::smem_desc(ghi + goff, 16, 1024), id1, ks > 0);
          sm100::mma_bf16(tmem + Lay::T_D1, a, sm100::smem_desc(glo + goff, 16, 1024), id1, true);
        }
        sm100::mma_bf16(tmem + Lay::T_D2, a, sm100::smem_desc(shi + ks * 2048, Lay::S_PANEL, 1024), id2, ks > 0);
        sm100::mma_bf16(tmem + Lay::T_D2, a, sm100::smem_desc(slo + ks * 2048, Lay::S_PANEL, 1024), id2, true);
      }
      sm100::mma_commit(&bar_mma);
    }
    if (!wait_all(&bar_mma, mma_phase)) { aborted = true; break; }
    mma_phase ^= 1;

    // ---------------------------------------------------------------- R = V - diag(A) K S0
    if (qw < 2) {
      const int i = row;  // token in chunk
      const float Ai = Aex[i];
#pragma unroll
      for (int cc = 0; cc < HALF; cc += 32) {
        const int c0 = ch * HALF + cc;
        float X[32];
        sm100::tmem_ld32(tmem + t_lane + Lay::T_D2 + c0, X);
        sm100::tmem_wait_ld();
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          const int cb = c0 + 8 * c8;
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            x[e] = ld_bf16(Vs + (cb / 64) * Lay::V_PANEL, sm100::sw128(i, (cb % 64) + e)) - Ai * X[8 * c8 + e];
          store8_split(Rhi, Rlo, (cb / 64) * Lay::RE_PANEL + sm100::sw128_chunk(i, (cb % 64) / 8), x);
        }
      }
    }
    __syncthreads();  // V is dead from here (Nf may alias it)

    // ---------------------------------------------------------------- N and Attn from D1
    {
      const int i = row & 63;
      const float li = ell[i];
      float X[32];
      sm100::tmem_ld32(tmem + t_lane + Lay::T_D1 + 32 * ch, X);
      sm100::tmem_wait_ld();
      if (qw < 2) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int j = 32 * ch + e;
          float v = 0.f;
          if (j < i) v = X[e] * __expf(li - ell[j]) * (VAR == kDelta ? sc2[j] : 1.f);
          Nf[fidx(i, j)] = v;
        }
      } else {
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int j = 32 * ch + 8 * c8 + e;
            x[e] = (j <= i) ? X[8 * c8 + e] * __expf(li - ell[j]) * (VAR == kDelta ? sc2[j] : 1.f) : 0.f;
          }
          store8_split(Thi, Tlo, sm100::sw128_chunk(64 + i, 4 * ch + c8), x);
        }
      }
    }
    __syncthreads();

    // ---------------------------------------------------------------- T = (I + N)^-1, blocked by 16
    if (tid < 64) {
      const int b = tid >> 4, cc = tid & 15;
      float t[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float acc = (i == cc) ? 1.f : 0.f;
#pragma unroll
        for (int j = 0; j < i; ++j) acc = fmaf(-Nf[fidx(16 * b + i, 16 * b + j)], t[j], acc);
        t[i] = acc;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) Tf[fidx(16 * b + i, 16 * b + cc)] = t[i];
    }
    __syncthreads();
#pragma unroll 1
    for (int d = 1; d < 4; ++d) {
      // M_ab = sum_{k=b}^{a-1} N_ak T_kb, kept in the (unused) upper block (b, a)
      for (int e = tid; e < (4 - d) * 256; e += kThreads) {
        const int b = e >> 8, a = b + d, ii = (e >> 4) & 15, jj = e & 15;
        float acc = 0.f;
        for (int k = b; k < a; ++k)
#pragma unroll
          for (int l = 0; l < 16; ++l) acc = fmaf(Nf[fidx(16 * a + ii, 16 * k + l)], Tf[fidx(16 * k + l, 16 * b + jj)], acc);
        Tf[fidx(16 * b + ii, 16 * a + jj)] = acc;
      }
      __syncthreads();
      // T_ab = -T_aa M_ab
      for (int e = tid; e < (4 - d) * 256; e += kThreads) {
        const int b = e >> 8, a = b + d, ii = (e >> 4) & 15, jj = e & 15;
        float acc = 0.f;
#pragma unroll
        for (int l = 0; l < 16; ++l) acc = fmaf(Tf[fidx(16 * a + ii, 16 * a + l)], Tf[fidx(16 * b + l, 16 * a + jj)], acc);
        Tf[fidx(16 * a + ii, 16 * b + jj)] = -acc;
      }
      __syncthreads();
    }
    {
      const int i = tid >> 2, q4 = tid & 3;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c8 = 2 * q4 + h;
        float x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int j = 8 * c8 + e;
          x[e] = (j < i) ? Tf[fidx(i, j)] : (j == i ? 1.f : 0.f);
        }
        store8_split(Thi, Tlo, sm100::sw128_chunk(i, c8), x);
      }
    }
    sm100::fence_async_smem();
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();

    const uint32_t thi = sm100::smem_u32(Thi), tlo = sm100::smem_u32(Tlo);
    // ---------------------------------------------------------------- DT = [T; Attn] T  (rows 64..127: AT)
    if (tid == 0) {
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
    if (!wait_all(&bar_mma, mma_phase)) { aborted = true; break; }
    mma_phase ^= 1;
    if (qw >= 2) {
      const int i = row - 64;
      float X[32];
      sm100::tmem_ld32(tmem + t_lane + Lay::T_DT + 32 * ch, X);
      sm100::tmem_wait_ld();
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        float x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = X[8 * c8 + e];
        store8_split(Thi, Tlo, sm100::sw128_chunk(64 + i, 4 * ch + c8), x);
      }
    }
    sm100::fence_async_smem();
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();

    // ---------------------------------------------------------------- D3 = [T; AT] R
    const uint32_t rhi = sm100::smem_u32(Rhi), rlo = sm100::smem_u32(Rlo);
    if (tid == 0) {
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
    if (!wait_all(&bar_mma, mma_phase)) { aborted = true; break; }
    mma_phase ^= 1;

    // ---------------------------------------------------------------- E -> scaled E panels, O out
    const float AC = Aex[kC - 1];
    if (qw < 2) {
      const int i = row;
      const float sc = __expf(ell[kC - 1] - ell[i]) * (VAR == kDelta ? sc2[i] : 1.f);  // A_C / A_i, no division
      float es = 0.f;
#pragma unroll
      for (int cc = 0; cc < HALF; cc += 32) {
        const int c0 = ch * HALF + cc;
        float X[32];
        sm100::tmem_ld32(tmem + t_lane + Lay::T_D3 + c0, X);
        sm100::tmem_wait_ld();
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          const int cb = c0 + 8 * c8;
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            es = fmaf(X[8 * c8 + e], X[8 * c8 + e], es);
            x[e] = X[8 * c8 + e] * sc;
          }
          store8_split(Rhi, Rlo, (cb / 64) * Lay::RE_PANEL + sm100::sw128_chunk(i, (cb % 64) / 8), x);
        }
      }
      en[ch][i] = es;
    } else {
      const int i = row - 64;
      const int tok = t0 + i;
      const float Ai = Aex[i];
#pragma unroll
      for (int cc = 0; cc < HALF; cc += 32) {
        const int c0 = ch * HALF + cc;
        float Y[32], Oi[32];
        sm100::tmem_ld32(tmem + t_lane + Lay::T_D2 + c0, Y);
        sm100::tmem_ld32(tmem + t_lane + Lay::T_D3 + c0, Oi);
        sm100::tmem_wait_ld();
        if (tok < L) {
          const size_t off = ((size_t)bh * L + tok) * D + c0;
          if (P.out_dtype == kF32) {
            float* op = reinterpret_cast<float*>(P.o) + off;
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(op + e) = make_float4(fmaf(Ai, Y[e], Oi[e]), fmaf(Ai, Y[e + 1], Oi[e + 1]),
                                                               fmaf(Ai, Y[e + 2], Oi[e + 2]), fmaf(Ai, Y[e + 3], Oi[e + 3]));
          } else {
            __nv_bfloat16* op = reinterpret_cast<__nv_bfloat16*>(P.o) + off;
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              __align__(16) __nv_bfloat16 h[8];
#pragma unroll
              for (int u = 0; u < 8; ++u) h[u] = __float2bfloat16_rn(fmaf(Ai, Y[e + u], Oi[e + u]));
              *reinterpret_cast<uint4*>(op + e) = *reinterpret_cast<const uint4*>(h);
            }
          }
        }
      }
    }
    sm100::fence_async_smem();
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    if (tid < kC && P.m != nullptr && t0 + tid < L)
      P.m[(size_t)bh * L + t0 + tid] = sqrtf(gn[tid]) * sqrtf(en[0][tid] + en[1][tid]);

    // ---------------------------------------------------------------- D4 = G^T Et
    if (tid == 0) {
      constexpr uint32_t id = sm100::idesc_bf16(128, D, true, true);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t bh_ = sm100::smem_desc(rhi + ks * 2048, Lay::RE_PANEL, 1024);
        const uint64_t bl = sm100::smem_desc(rlo + ks * 2048, Lay::RE_PANEL, 1024);
        if (VAR == kDelta) {
          const uint64_t ak = sm100::smem_desc(kq0 + ks * 2048, Lay::KQ_PANEL, 1024);
          sm100::mma_bf16(tmem + Lay::T_D4, ak, bh_, id, ks > 0);
          sm100::mma_bf16(tmem + Lay::T_D4, ak, bl, id, true);
        } else {
          const uint64_t ah = sm100::smem_desc(sm100::smem_u32(Ghi) + ks * 2048, Lay::G_PANEL, 1024);
          const uint64_t al = sm100::smem_desc(sm100::smem_u32(Glo) + ks * 2048, Lay::G_PANEL, 1024);
          sm100::mma_bf16(tmem + Lay::T_D4, ah, bh_, id, ks > 0);
          sm100::mma_bf16(tmem + Lay::T_D4, al, bh_, id, true);
          sm100::mma_bf16(tmem + Lay::T_D4, ah, bl, id, true);
        }
      }
      sm100::mma_commit(&bar_mma);
    }
    if (!wait_all(&bar_mma, mma_phase)) { aborted = true; break; }
    mma_phase ^= 1;

    // ---------------------------------------------------------------- S <- A_C S + D4
    if (s_owner) {
#pragma unroll
      for (int cc = 0; cc < HALF; cc += 32) {
        float X[32];
        sm100::tmem_ld32(tmem + t_lane + Lay::T_D4 + ch * HALF + cc, X);
        sm100::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) Sr[cc + e] = fmaf(AC, Sr[cc + e], X[e]);
      }
    }
    write_state_panels();
    sm100::fence_async_smem();
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
  }

  // ---- write back the state (and the diagonal covariance)
  if (!aborted) {
    if (s_owner) {
#pragma unroll
      for (int c = 0; c < HALF; c += 4)
        *reinterpret_cast<float4*>(Sg + (size_t)row * D + ch * HALF + c) =
            make_float4(Sr[c], Sr[c + 1], Sr[c + 2], Sr[c + 3]);
    }
    if (VAR == kDiag && pi >= 0 && pi < D) P.p[(size_t)bh * D + pi] = pcur;
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
bool make_tmap(CUtensorMap* tm, const void* base, int BH, int L, int d) {
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

bool chunk_supported(kdn_variant variant, const kdn_dims& d) {
  (void)variant;
  return d.in_dtype == KDN_BF16 && d.dk == d.dv && (d.dk == 64 || d.dk == 128) && (d.chunk == 0 || d.chunk == 64) &&
         d.L > 0 && encode_fn() != nullptr;
}

void chunk_plan(kdn_variant variant, const kdn_dims&, int* launches, const char** kernel, const char** arith) {
  *launches = variant == KDN_KALMAN_FULL ? 2 : 1;
  *kernel = variant == KDN_KALMAN_FULL ? "kalman_full_gains_kernel" : "chunk_scan_kernel";
  *arith = "bf16-tc";
}

cudaError_t launch_chunk(kdn_variant variant, const kdn_dims& d, const ChunkArgs& a, cudaStream_t stream) {
  const int BH = a.BH;
  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, a.q, BH, a.L, d.dk) || !make_tmap(&tk, a.k, BH, a.L, d.dk) || !make_tmap(&tv, a.v, BH, a.L, d.dv))
    return cudaErrorInvalidValue;
  Params p{};
  p.beta = a.beta, p.a = a.a, p.r = a.r, p.qn = a.qn, p.qn_scalar = a.qn_scalar;
  p.S = a.S, p.o = a.o, p.m = a.m, p.out_dtype = a.out_dtype, p.L = a.L, p.status = a.status;
  if (variant == KDN_KALMAN_FULL) {
    // covariance side first: per-token gains into the workspace, then the chunked S side
    float* gains = reinterpret_cast<float*>(a.workspace);
    GainArgs g{a.k, KDN_BF16, a.a, a.r, a.qn, a.qn_scalar, a.P, nullptr, gains, a.status, BH, a.L};
    cudaError_t e = launch_kalman_full_gains(d.dk, g, stream);
    if (e != cudaSuccess) return e;
    p.gains = gains;
    return d.dk == 64 ? launch_typed<64, kFull>(tq, tk, tv, p, BH, stream)
                      : launch_typed<128, kFull>(tq, tk, tv, p, BH, stream);
  }
  if (variant == KDN_KALMAN_DIAG) {
    p.p = a.P;
    return d.dk == 64 ? launch_typed<64, kDiag>(tq, tk, tv, p, BH, stream)
                      : launch_typed<128, kDiag>(tq, tk, tv, p, BH, stream);
  }
  return d.dk == 64 ? launch_typed<64, kDelta>(tq, tk, tv, p, BH, stream)
                    : launch_typed<128, kDelta>(tq, tk, tv, p, BH, stream);
}

}  // namespace kdn
