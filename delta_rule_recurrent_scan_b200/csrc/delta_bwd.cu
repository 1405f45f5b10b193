// Backward pass of the gated delta rule scan (the training-time adjoint), on the fp32 CUDA cores.
//
// Forward, per head (A Hippocampus for Linear Attention, section 3.3 Eq. (5)-(6) and section 3.5):
//   e_t = v_t - a_t S_{t-1}^T k_t,  S_t = a_t S_{t-1} + beta_t k_t e_t^T,  o_t = S_t^T q_t,
//   m_t = beta_t ||k_t|| ||e_t||.
// The pages train these layers end to end (same page, section 4; Kalman Delta Networks, Abstract) but
// print no backward.  This is the adjoint of the chunk form (chunks of kCB tokens, gates restarting at
// every chunk start: ell_i = sum_{m<=i} log a_m, A_i = exp(ell_i), Gam_ij = exp(ell_i - ell_j), i >= j,
// r_j = A_C / A_j, G = diag(beta) K):
//   N = strict_lower((K G^T) o Gam), T = (I + N)^-1, M = lower((Q G^T) o Gam), AT = M T,
//   R = V - diag(A) K S0, E = T R, O = diag(A) Q S0 + AT R, S_C = A_C S0 + G^T diag(r) E.
// Walking the chunks backwards with the state adjoint dS (dLoss/dS_C), every step is a product of
// C x C, C x d or d x d blocks:
//   dE = diag(r) G dS (+ the surprise term), dW = dS E^T, dAT = dO R^T, dR = AT^T dO + T^T dE,
//   dT = dE R^T + M^T dAT, dM = lower(dAT T^T), dN = strict_lower(-T^T dT T^T),
//   dKG = dN o Gam, dQG = dM o Gam, dGam = dN o KG + dM o QG,
//   dq = diag(A) dO S0^T + dQG G,  dk = -diag(A) dR S0^T + dKG G + diag(beta) dG,  dv = dR,
//   dG = dKG^T K + dQG^T Q + diag(r) dW^T,  dbeta_i = k_i . dG_i,
//   dS0 = A_C dS + Q^T diag(A) dO - K^T diag(A) dR  (the previous chunk's dS).
// Gate gradients are taken without dividing by a gate (a_t = 0, a full reset, is allowed): every
// derivative of a product of gates by a_t is the product of the other gates, e.g.
// dA_i / da_t = A_{t-1} Gam_it (t <= i), dGam_ij / da_t = Gam_it Gam_{t-1,j} (j < t <= i),
// dr_j / da_t = Gam_{t-1,j} Gam_{C-1,t} (j < t), and the sums over j < t run as prefix recursions
// H_{t+1} = a_t H_t + x_t.
//
// Work split: one CTA per (head, block of 32 value columns).  The columns of S evolve independently,
// so dS, dv and dS0 of a column block are its own; dq, dk, dbeta and da are sums over the column
// blocks and are added into the (zeroed) outputs with atomics.  The chunk-start states come from a
// forward pass that writes them every kCB tokens, with the residual norms ||e_t|| the surprise
// gradient needs (they span all columns).
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace kdn {

namespace {

constexpr int kCB = 32;          // tokens per backward chunk (and between forward checkpoints)
constexpr int kJB = 32;          // value columns per CTA
constexpr int kBwdThreads = 512;
constexpr float kLogFloor = -60.f;  // a gate of 0 enters the logs as exp(-60), as in the forward

// C[i][j] (row stride ldc) = alpha * sum_k A(i,k) B(k,j) (+ C[i][j] when acc), for i < M, j < N, with
// A(i,k) = A[i ai + k ak] and B(k,j) = B[k bk + j bj] in shared memory (C aliases neither).  Each thread
// takes a TM x TN register tile (TM + TN loads per TM TN multiply-adds); when the tiles are fewer than the
// threads, S adjacent lanes share a tile, each summing every S-th k, and their parts are summed by shuffles
// (TILES S is then a multiple of 32 and at most the block, so every lane of a warp takes part).  Ends with
// a barrier.
template <int M, int N, int K, int TM, int TN>
__device__ __forceinline__ void mm(float* C, int ldc, const float* A, int ai, int ak, const float* B, int bk, int bj,
                                   float alpha, bool acc) {
  static_assert(M % TM == 0 && N % TN == 0, "tile");
  constexpr int NTI = N / TN, TILES = (M / TM) * NTI;
  constexpr int S0 = kBwdThreads / TILES < 1 ? 1 : kBwdThreads / TILES;
  constexpr int S = S0 >= 8 && K % 8 == 0 ? 8 : S0 >= 4 && K % 4 == 0 ? 4 : S0 >= 2 && K % 2 == 0 ? 2 : 1;
  static_assert(S == 1 || (TILES * S % 32 == 0 && TILES * S <= kBwdThreads), "whole warps share the tiles");
  for (int item = threadIdx.x; item < TILES * S; item += kBwdThreads) {
    const int sp = item % S, tile = item / S;
    const int i0 = (tile / NTI) * TM, j0 = (tile % NTI) * TN;
    float s[TM][TN];
#pragma unroll
    for (int u = 0; u < TM; ++u)
#pragma unroll
      for (int w = 0; w < TN; ++w) s[u][w] = 0.f;
#pragma unroll 4
    for (int k = sp; k < K; k += S) {
      float av[TM], bv[TN];
#pragma unroll
      for (int u = 0; u < TM; ++u) av[u] = A[(i0 + u) * ai + k * ak];
#pragma unroll
      for (int w = 0; w < TN; ++w) bv[w] = B[k * bk + (j0 + w) * bj];
#pragma unroll
      for (int u = 0; u < TM; ++u)
#pragma unroll
        for (int w = 0; w < TN; ++w) s[u][w] = fmaf(av[u], bv[w], s[u][w]);
    }
#pragma unroll
    for (int o = S / 2; o > 0; o >>= 1)
#pragma unroll
      for (int u = 0; u < TM; ++u)
#pragma unroll
        for (int w = 0; w < TN; ++w) s[u][w] += __shfl_xor_sync(0xffffffffu, s[u][w], o);
    if (sp == 0) {
#pragma unroll
      for (int u = 0; u < TM; ++u)
#pragma unroll
        for (int w = 0; w < TN; ++w) {
          float* c = C + (i0 + u) * ldc + j0 + w;
          *c = acc ? fmaf(alpha, s[u][w], *c) : alpha * s[u][w];
        }
    }
  }
  __syncthreads();
}

// Shared-memory layout of one CTA for JB value columns (floats; every row padded by one so that walks down
// a column avoid bank conflicts).
template <int DK, int JB, bool GEN>
struct BwdSmem {
  static constexpr int LK = DK + 1, LJ = JB + 1, LC = kCB + 1;
  static constexpr int KC = 0;                    // K of the chunk [kCB][LK]
  static constexpr int QC = KC + kCB * LK;        // Q
  static constexpr int S0 = QC + kCB * LK;        // chunk-start state, this CTA's columns [DK][LJ]
  static constexpr int DS = S0 + DK * LJ;         // state adjoint [DK][LJ]
  static constexpr int VC = DS + DK * LJ;         // [kCB][LJ] blocks: V, dO (then diag(A) dO), KS, QS,
  static constexpr int DO = VC + kCB * LJ;        //   R, E, dE, dR (then -diag(A) dR)
  static constexpr int KS = DO + kCB * LJ;
  static constexpr int QS = KS + kCB * LJ;
  static constexpr int RR = QS + kCB * LJ;
  static constexpr int EE = RR + kCB * LJ;
  static constexpr int DE = EE + kCB * LJ;
  static constexpr int DR = DE + kCB * LJ;
  static constexpr int GAM = DR + kCB * LJ;       // [kCB][LC] blocks
  static constexpr int KG = GAM + kCB * LC;       // K G^T (with beta_j)
  static constexpr int QG = KG + kCB * LC;        // Q G^T
  static constexpr int TT = QG + kCB * LC;        // T = (I + N)^-1
  static constexpr int MM = TT + kCB * LC;        // M
  static constexpr int AT = MM + kCB * LC;        // AT = M T
  static constexpr int DAT = AT + kCB * LC;       // dAT, later T^T dT
  static constexpr int DT = DAT + kCB * LC;       // dT
  static constexpr int DM = DT + kCB * LC;        // dM, then dQG
  static constexpr int DN = DM + kCB * LC;        // dN, then dKG
  static constexpr int DW = DN + kCB * LC;        // dW = dS E^T [DK][LC]
  static constexpr int VEC = DW + DK * LC;        // per-token vectors of kCB floats (see the kernel)
  static constexpr int NVEC = 12;
  static constexpr int GC = VEC + NVEC * kCB + 32; // general gains: the chunk's G [kCB][LK]
  static constexpr int RAW = (GC + (GEN ? kCB * LK : 0) + 3) / 4 * 4;  // the next chunk's inputs as copied
  // raw stage (in floats from RAW): K, Q [kCB][DK] and V [kCB][JB] as bf16 (fp32 inputs are read directly),
  // dO [kCB][JB], S0 [DK][JB], then a, beta, dm and ||e|| [kCB] each
  static constexpr int RK = 0, RQ = RK + kCB * DK / 2, RV = RQ + kCB * DK / 2, RO = RV + kCB * JB / 2;
  static constexpr int RS = RO + kCB * JB;
  static constexpr int RA = RS + DK * JB, RB = RA + kCB, RM = RB + kCB, RE = RM + kCB, RAW_FLOATS = RE + kCB;
  static constexpr int TOTAL = RAW + RAW_FLOATS;
  static constexpr size_t BYTES = TOTAL * sizeof(float);
};

// GEN: the gains are given per token (g_t, a d_k vector: diagonal Kalman) instead of beta_t k_t, and dG is
// written instead of dbeta (the key then carries no gain term).
template <int DK, int DV, bool GEN>
__global__ void __launch_bounds__(kBwdThreads, 1) delta_bwd_kernel(DeltaBwdArgs p) {
  constexpr int JB = DV < kJB ? DV : kJB;
  using Lay = BwdSmem<DK, JB, GEN>;
  constexpr int LK = Lay::LK, LJ = Lay::LJ, LC = Lay::LC, C = kCB, NT = kBwdThreads, NW = NT / 32;
  extern __shared__ float sm[];
  float* Kc = sm + Lay::KC;
  float* Qc = sm + Lay::QC;
  float* S0 = sm + Lay::S0;
  float* dS = sm + Lay::DS;
  float* Vc = sm + Lay::VC;
  float* dOc = sm + Lay::DO;
  float* KS = sm + Lay::KS;
  float* QS = sm + Lay::QS;
  float* Rr = sm + Lay::RR;
  float* Ee = sm + Lay::EE;
  float* dE = sm + Lay::DE;
  float* dR = sm + Lay::DR;
  float* Gam = sm + Lay::GAM;
  float* KG = sm + Lay::KG;
  float* QG = sm + Lay::QG;
  float* Tt = sm + Lay::TT;
  float* Mm = sm + Lay::MM;
  float* AT = sm + Lay::AT;
  float* dAT = sm + Lay::DAT;
  float* dT = sm + Lay::DT;
  float* dM = sm + Lay::DM;
  float* dN = sm + Lay::DN;
  float* dW = sm + Lay::DW;
  float* vec = sm + Lay::VEC;
  float* va = vec;             // gate a_t as used (a gate of 0 floored like the log)
  float* vb = vec + C;         // beta
  float* vell = vec + 2 * C;   // ell
  float* vA = vec + 3 * C;     // A
  float* vr = vec + 4 * C;     // r = A_C / A
  float* vdm = vec + 5 * C;    // dLoss/dm
  float* ven = vec + 6 * C;    // ||e|| (all columns, from the forward)
  float* vkn = vec + 7 * C;    // ||k|| (||g|| for given gains)
  float* Gc = sm + Lay::GC;    // given gains of the chunk (GEN)
  float* vdA = vec + 8 * C;    // dLoss/dA (this block's columns)
  float* vdr = vec + 9 * C;    // dLoss/dr
  float* vdb = vec + 10 * C;   // dbeta
  float* vh = vec + 11 * C;    // prefix sums of the r term
  float* vmisc = vec + 12 * C; // [0]: dLoss/dA_C

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x, j0 = blockIdx.y * JB;
  const int L = p.L, nck = (L + C - 1) / C;
  const size_t tok0 = (size_t)bh * L;
  const bool first_block = blockIdx.y == 0;  // adds the surprise terms that span all columns

  for (int idx = tid; idx < DK * JB; idx += NT) {
    const int kk = idx / JB, j = idx % JB;
    dS[kk * LJ + j] = p.dS_L != nullptr ? p.dS_L[((size_t)bh * DK + kk) * DV + j0 + j] : 0.f;
  }

  // The inputs of chunk c - 1 are copied asynchronously into the raw stage while chunk c is worked on (the
  // walk is backwards); each chunk starts by spreading its stage into the padded working layouts.
  float* raw = sm + Lay::RAW;
  const bool raw_in = p.in_dtype == kBF16;  // bf16 keys, queries, values go through the stage
  auto issue = [&](int cc) {
    if (cc >= 0) {
      const int u0 = cc * C, nn = min(C, L - u0);
      const int och = JB * 4 / 16;  // 16-byte pieces of one fp32 row's column block
      if (raw_in) {
        const uint8_t* kb = static_cast<const uint8_t*>(p.k) + (tok0 + u0) * DK * 2;
        const uint8_t* qb = static_cast<const uint8_t*>(p.q) + (tok0 + u0) * DK * 2;
        async_copy_rows(raw + Lay::RK, kb, nn * DK * 2, tid, NT);
        async_copy_rows(raw + Lay::RQ, qb, nn * DK * 2, tid, NT);
        const int vch = JB * 2 / 16;
        for (int idx = tid; idx < nn * vch; idx += NT) {
          const int i = idx / vch, q = idx % vch;
          async_copy16(reinterpret_cast<uint8_t*>(raw + Lay::RV) + (size_t)i * JB * 2 + 16 * q,
                       static_cast<const uint8_t*>(p.v) + ((tok0 + u0 + i) * DV + j0) * 2 + 16 * q);
        }
      }
      for (int idx = tid; idx < nn * och; idx += NT) {
        const int i = idx / och, q = idx % och;
        async_copy16(raw + Lay::RO + i * JB + 4 * q, p.dO + (tok0 + u0 + i) * DV + j0 + 4 * q);
      }
      for (int idx = tid; idx < DK * och; idx += NT) {
        const int kk = idx / och, q = idx % och;
        async_copy16(raw + Lay::RS + kk * JB + 4 * q, p.S_ckpt + (((size_t)bh * nck + cc) * DK + kk) * DV + j0 + 4 * q);
      }
      if (tid < nn) {
        const size_t ti = tok0 + u0 + tid;
        if (p.a != nullptr) async_copy4(raw + Lay::RA + tid, p.a + ti); else raw[Lay::RA + tid] = 1.f;
        if (!GEN) async_copy4(raw + Lay::RB + tid, p.beta + ti); else raw[Lay::RB + tid] = 1.f;
        if (p.dm != nullptr) async_copy4(raw + Lay::RM + tid, p.dm + ti); else raw[Lay::RM + tid] = 0.f;
        async_copy4(raw + Lay::RE + tid, p.enorm + ti);
      }
    }
    async_commit();
  };
  auto raw_bf16 = [&](int off, int idx) { return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(raw + off)[idx]); };
  issue(nck - 1);

  for (int c = nck - 1; c >= 0; --c) {
    const int t0 = c * C, n = min(C, L - t0);
    async_wait<0>();
    __syncthreads();  // this chunk's inputs are in, and the previous chunk is done with every buffer
    // ------------------------------------------------------------------ inputs of the chunk (zero past L)
    for (int idx = tid; idx < C * DK; idx += NT) {
      const int i = idx / DK, kk = idx % DK;
      const bool ok = i < n;
      const size_t off = (tok0 + t0 + i) * DK + kk;
      Kc[i * LK + kk] = ok ? (raw_in ? raw_bf16(Lay::RK, idx) : load_elem(p.k, off, p.in_dtype)) : 0.f;
      Qc[i * LK + kk] = ok ? (raw_in ? raw_bf16(Lay::RQ, idx) : load_elem(p.q, off, p.in_dtype)) : 0.f;
      if (GEN) Gc[i * LK + kk] = ok ? p.gains[off] : 0.f;
    }
    for (int idx = tid; idx < C * JB; idx += NT) {
      const int i = idx / JB, j = idx % JB;
      const bool ok = i < n;
      Vc[i * LJ + j] = ok ? (raw_in ? raw_bf16(Lay::RV, idx) : load_elem(p.v, (tok0 + t0 + i) * DV + j0 + j, p.in_dtype))
                          : 0.f;
      dOc[i * LJ + j] = ok ? raw[Lay::RO + idx] : 0.f;
    }
    for (int idx = tid; idx < DK * JB; idx += NT) S0[(idx / JB) * LJ + idx % JB] = raw[Lay::RS + idx];
    if (tid < C) {
      const int i = tid;
      const bool ok = i < n;
      va[i] = ok ? raw[Lay::RA + i] : 1.f;
      vb[i] = GEN ? 1.f : (ok ? raw[Lay::RB + i] : 0.f);
      vdm[i] = ok ? raw[Lay::RM + i] : 0.f;
      ven[i] = ok ? raw[Lay::RE + i] : 0.f;
      vdA[i] = 0.f, vdr[i] = 0.f, vdb[i] = 0.f;
    }
    if (tid == 0) vmisc[0] = 0.f;
    __syncthreads();
    issue(c - 1);  // the stage is free again
    // ------------------------------------------------------------------ gates (warp 0), key norms (all warps)
    if (warp == 0) {
      // ell (for the ratios Gam_ij = exp(ell_i - ell_j), a gate of 0 floored at e^-60 there), and A_i, r_j as
      // exact prefix and suffix products of the gates, so that a reset zeroes them exactly (dS0 and the
      // terms through diag(A) then vanish as in the token recurrence)
      const float a = va[lane];
      float x = a > 0.f ? fmaxf(__logf(a), kLogFloor) : kLogFloor;
      va[lane] = __expf(x);  // the gate in the prefix recursions of the gate gradient
      float pa = a, sa = a;  // inclusive prefix product, exclusive suffix product (below)
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o), py = __shfl_up_sync(0xffffffffu, pa, o);
        if (lane >= o) x += y, pa *= py;
      }
      const float a_next = __shfl_down_sync(0xffffffffu, a, 1);  // every lane takes part in the shuffle
      sa = lane < C - 1 ? a_next : 1.f;                            // a_{j+1}
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_down_sync(0xffffffffu, sa, o);
        if (lane + o < C) sa *= y;  // prod_{m > j} a_m
      }
      vell[lane] = x;
      vA[lane] = pa;
      vr[lane] = sa;
    }
    for (int i = warp; i < C; i += NW) {
      const float* rowv = GEN ? Gc : Kc;
      float sq = 0.f;
      for (int kk = lane; kk < DK; kk += 32) sq = fmaf(rowv[i * LK + kk], rowv[i * LK + kk], sq);
      sq = warp_sum(sq);
      if (lane == 0) vkn[i] = sqrtf(sq);
    }
    __syncthreads();
    for (int idx = tid; idx < C * C; idx += NT) {
      const int i = idx / C, j = idx % C;
      Gam[i * LC + j] = j <= i ? __expf(vell[i] - vell[j]) : 0.f;
    }
    // ------------------------------------------------------------------ forward recompute of the chunk
    mm<C, C, DK, 4, 4>(KG, LC, Kc, LK, 1, GEN ? Gc : Kc, 1, LK, 1.f, false);  // K K^T (K G^T)
    mm<C, C, DK, 4, 4>(QG, LC, Qc, LK, 1, GEN ? Gc : Kc, 1, LK, 1.f, false);  // Q K^T (Q G^T)
    for (int idx = tid; idx < C * C; idx += NT) {
      const int i = idx / C, j = idx % C;
      const float kg = KG[i * LC + j] * vb[j], qg = QG[i * LC + j] * vb[j], g = Gam[i * LC + j];
      KG[i * LC + j] = kg, QG[i * LC + j] = qg;
      Mm[i * LC + j] = j <= i ? qg * g : 0.f;
      dN[i * LC + j] = j < i ? kg * g : 0.f;  // N, scratch until the backward needs dN
    }
    __syncthreads();
    if (tid < C) {  // T = (I + N)^-1 by columns: t_i = delta_ic - sum_{m < i} N_im t_m
      const int cc = tid;
      float t[C];
#pragma unroll
      for (int i = 0; i < C; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < i; ++m) acc = fmaf(dN[i * LC + m], t[m], acc);
        t[i] = (i == cc) ? 1.f : -acc;  // rows above cc stay 0: every t_m with m < cc is 0
        if (i < cc) t[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < C; ++i) Tt[i * LC + cc] = t[i];
    }
    __syncthreads();
    mm<C, C, C, 2, 2>(AT, LC, Mm, LC, 1, Tt, LC, 1, 1.f, false);
    mm<C, JB, DK, 4, 4>(KS, LJ, Kc, LK, 1, S0, LJ, 1, 1.f, false);
    mm<C, JB, DK, 4, 4>(QS, LJ, Qc, LK, 1, S0, LJ, 1, 1.f, false);
    for (int idx = tid; idx < C * JB; idx += NT) {
      const int i = idx / JB, j = idx % JB;
      Rr[i * LJ + j] = Vc[i * LJ + j] - vA[i] * KS[i * LJ + j];
    }
    __syncthreads();
    mm<C, JB, C, 2, 2>(Ee, LJ, Tt, LC, 1, Rr, LJ, 1, 1.f, false);  // E = T R
    // ------------------------------------------------------------------ backward of the chunk
    mm<C, JB, DK, 4, 4>(dE, LJ, GEN ? Gc : Kc, LK, 1, dS, LJ, 1, 1.f, false);  // K dS (G dS)
    {
      float acc = 0.f;  // dLoss/dA_C from S_C = A_C S0 + ...: this block's sum of dS o S0
      for (int idx = tid; idx < DK * JB; idx += NT) {
        const int kk = idx / JB, j = idx % JB;
        acc = fmaf(dS[kk * LJ + j], S0[kk * LJ + j], acc);
      }
      acc = warp_sum(acc);
      if (lane == 0) atomicAdd(&vmisc[0], acc);
    }
    for (int idx = tid; idx < C * JB; idx += NT) {
      const int i = idx / JB, j = idx % JB;
      float de = vr[i] * vb[i] * dE[i * LJ + j];
      if (ven[i] > 0.f) de = fmaf(vdm[i] * vb[i] * vkn[i] / ven[i], Ee[i * LJ + j], de);  // d m / d e
      dE[i * LJ + j] = de;
    }
    __syncthreads();
    mm<DK, C, JB, 4, 4>(dW, LC, dS, LJ, 1, Ee, 1, LJ, 1.f, false);           // dW = dS E^T
    mm<C, C, JB, 2, 2>(dAT, LC, dOc, LJ, 1, Rr, 1, LJ, 1.f, false);          // dAT = dO R^T
    mm<C, JB, C, 2, 2>(dR, LJ, AT, 1, LC, dOc, LJ, 1, 1.f, false);           // dR = AT^T dO
    mm<C, JB, C, 2, 2>(dR, LJ, Tt, 1, LC, dE, LJ, 1, 1.f, true);             //    + T^T dE
    mm<C, C, JB, 2, 2>(dT, LC, dE, LJ, 1, Rr, 1, LJ, 1.f, false);           // dT = dE R^T
    mm<C, C, C, 2, 2>(dT, LC, Mm, 1, LC, dAT, LC, 1, 1.f, true);             //    + M^T dAT
    mm<C, C, C, 2, 2>(dM, LC, dAT, LC, 1, Tt, 1, LC, 1.f, false);            // dM = dAT T^T (masked below)
    mm<C, C, C, 2, 2>(dAT, LC, Tt, 1, LC, dT, LC, 1, 1.f, false);            // X = T^T dT (over dAT)
    mm<C, C, C, 2, 2>(dN, LC, dAT, LC, 1, Tt, 1, LC, -1.f, false);           // dN = -X T^T (masked below)
    for (int idx = tid; idx < C * C; idx += NT) {
      const int i = idx / C, j = idx % C;
      const float dn = j < i ? dN[i * LC + j] : 0.f, dmv = j <= i ? dM[i * LC + j] : 0.f, g = Gam[i * LC + j];
      dT[i * LC + j] = dn * KG[i * LC + j] + dmv * QG[i * LC + j];  // dGam
      dN[i * LC + j] = dn * g;                                         // dKG = d(K G^T)
      dM[i * LC + j] = dmv * g;                                        // dQG = d(Q G^T)
    }
    // dA (this block's part): diag(A) enters through Q S0 and K S0
    for (int i = warp; i < C; i += NW) {
      float acc = 0.f;
      for (int j = lane; j < JB; j += 32)
        acc += dOc[i * LJ + j] * QS[i * LJ + j] - dR[i * LJ + j] * KS[i * LJ + j];
      acc = warp_sum(acc);
      if (lane == 0) vdA[i] = acc;
    }
    __syncthreads();
    // dv = dR; then dQS = diag(A) dO and dKS = -diag(A) dR in place
    for (int idx = tid; idx < C * JB; idx += NT) {
      const int i = idx / JB, j = idx % JB;
      if (i < n) p.dv[(tok0 + t0 + i) * DV + j0 + j] = dR[i * LJ + j];
      dOc[i * LJ + j] *= vA[i];
      dR[i * LJ + j] *= -vA[i];
    }
    __syncthreads();
    // ------------------------------------------------------------------ dq, dk, dG, dbeta (C x DK)
    // dq_ik = sum_j dQS_ij S0_kj + sum_m dQG_im beta_m K_mk
    // dk_ik = sum_j dKS_ij S0_kj + sum_m dKG_im beta_m K_mk + beta_i dG_ik
    // dG_ik = sum_m dKG_mi K_mk + sum_m dQG_mi Q_mk + r_i dW_ki (+ the surprise term, first block)
    // Thread: tokens i0, i0 + 1 and the four columns kk = kq + (DK / 4) e (a warp reads 32 consecutive
    // columns of a row at a time).
    {
      constexpr int KQ = DK / 4, SEG = KQ < 32 ? KQ : 32;  // lanes that share a token pair
      for (int item = tid; item < (C / 2) * KQ; item += NT) {
        const int i0 = 2 * (item / KQ), kq = item % KQ;
        float dq[2][4], dk[2][4], dg[2][4];
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int e = 0; e < 4; ++e) dq[a][e] = dk[a][e] = dg[a][e] = 0.f;
#pragma unroll 4
        for (int j = 0; j < JB; ++j) {
          const float o0 = dOc[i0 * LJ + j], o1 = dOc[(i0 + 1) * LJ + j];
          const float r0 = dR[i0 * LJ + j], r1 = dR[(i0 + 1) * LJ + j];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float s0 = S0[(kq + KQ * e) * LJ + j];
            dq[0][e] = fmaf(o0, s0, dq[0][e]), dq[1][e] = fmaf(o1, s0, dq[1][e]);
            dk[0][e] = fmaf(r0, s0, dk[0][e]), dk[1][e] = fmaf(r1, s0, dk[1][e]);
          }
        }
#pragma unroll 4
        for (int m = 0; m < C; ++m) {
          const float bm = vb[m];
          const float qa0 = dM[i0 * LC + m] * bm, qa1 = dM[(i0 + 1) * LC + m] * bm;
          const float ka0 = dN[i0 * LC + m] * bm, ka1 = dN[(i0 + 1) * LC + m] * bm;
          const float gk0 = dN[m * LC + i0], gk1 = dN[m * LC + i0 + 1];
          const float gq0 = dM[m * LC + i0], gq1 = dM[m * LC + i0 + 1];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float km = Kc[m * LK + kq + KQ * e], qm = Qc[m * LK + kq + KQ * e];
            const float gm = GEN ? Gc[m * LK + kq + KQ * e] : km;  // the gain row (beta_m enters through bm)
            dq[0][e] = fmaf(qa0, gm, dq[0][e]), dq[1][e] = fmaf(qa1, gm, dq[1][e]);
            dk[0][e] = fmaf(ka0, gm, dk[0][e]), dk[1][e] = fmaf(ka1, gm, dk[1][e]);
            dg[0][e] = fmaf(gk0, km, fmaf(gq0, qm, dg[0][e]));
            dg[1][e] = fmaf(gk1, km, fmaf(gq1, qm, dg[1][e]));
          }
        }
        float db[2];
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          const int i = i0 + a;
          const float sur = first_block && vkn[i] > 0.f ? vdm[i] * ven[i] / vkn[i] : 0.f;
          db[a] = 0.f;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int kk = kq + KQ * e;
            const float ki = Kc[i * LK + kk];
            float g = fmaf(vr[i], dW[kk * LC + i], dg[a][e]);
            g = fmaf(sur, GEN ? Gc[i * LK + kk] : ki, g);  // the surprise along the gain's direction
            if (!GEN) dk[a][e] = fmaf(vb[i], g, dk[a][e]);
            db[a] = fmaf(ki, g, db[a]);  // dbeta_i = k_i . dG_i
            dg[a][e] = g;
          }
          if (i < n) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const size_t off = (tok0 + t0 + i) * DK + kq + KQ * e;
              atomicAdd(p.dq + off, dq[a][e]);
              atomicAdd(p.dk + off, dk[a][e]);
              if (GEN) atomicAdd(p.dgain + off, dg[a][e]);
            }
          }
        }
        // the token pair's SEG lanes sum their columns' parts (every lane of a warp is here: (C / 2) KQ is a
        // multiple of 32)
#pragma unroll
        for (int o = SEG / 2; o > 0; o >>= 1) {
          db[0] += __shfl_xor_sync(0xffffffffu, db[0], o);
          db[1] += __shfl_xor_sync(0xffffffffu, db[1], o);
        }
        if (lane % SEG == 0) atomicAdd(&vdb[i0], db[0]), atomicAdd(&vdb[i0 + 1], db[1]);
      }
    }
    // dLoss/dr_j = beta_j sum_k K_jk dW_kj (sum_k G_jk dW_kj for given gains)
    for (int j = warp; j < C; j += NW) {
      const float* rowv = GEN ? Gc : Kc;
      float acc = 0.f;
      for (int kk = lane; kk < DK; kk += 32) acc = fmaf(rowv[j * LK + kk], dW[kk * LC + j], acc);
      acc = warp_sum(acc);
      if (lane == 0) vdr[j] = vb[j] * acc;
    }
    __syncthreads();
    // ------------------------------------------------------------------ gate gradients (this block's part)
    // da_t = A_{t-1} sum_{i>=t} Gam_it dA_i + sum_{i>=t} Gam_it H_it + Gam_{C-1,t} h_t + A_{t-1} Gam_{C-1,t} dA_C,
    // H_{i,t} = sum_{j<t} Gam_{t-1,j} dGam_ij (H_{i,t+1} = a_t H_{i,t} + dGam_it), h_t likewise for dr.
    // The H of row i (kept in dAT) and h run on one thread each.
    if (tid < C) {
      const int i = tid;
      float h = 0.f;
      for (int t = 0; t <= i; ++t) {
        dAT[i * LC + t] = h;
        h = fmaf(va[t], h, dT[i * LC + t]);
      }
    } else if (tid == C) {
      float h = 0.f;
      for (int t = 0; t < C; ++t) {
        vh[t] = h;
        h = fmaf(va[t], h, vdr[t]);
      }
    }
    __syncthreads();
    if (tid < C) {
      const int t = tid;
      float sA = 0.f, sH = 0.f;
      for (int i = t; i < C; ++i) {
        const float g = Gam[i * LC + t];
        sA = fmaf(g, vdA[i], sA);
        sH = fmaf(g, dAT[i * LC + t], sH);
      }
      const float Aprev = t > 0 ? vA[t - 1] : 1.f, gC = Gam[(C - 1) * LC + t];
      const float da = Aprev * sA + sH + gC * vh[t] + Aprev * gC * vmisc[0];
      if (t < n) {
        if (p.da != nullptr) atomicAdd(p.da + tok0 + t0 + t, da);
        if (!GEN) atomicAdd(p.dbeta + tok0 + t0 + t, vdb[t]);
      }
    }
    // ------------------------------------------------------------------ dS0 = A_C dS + Q^T dQS + K^T dKS, in place
    // thread: rows kk = kq + (DK / 4) e and columns j0, j0 + 1
    {
      constexpr int KQ = DK / 4, JP = JB / 2;
      const float AC = vA[C - 1];
      for (int item = tid; item < KQ * JP; item += NT) {
        const int kq = item / JP, jj = 2 * (item % JP);
        float acc[4][2];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[e][0] = AC * dS[(kq + KQ * e) * LJ + jj];
          acc[e][1] = AC * dS[(kq + KQ * e) * LJ + jj + 1];
        }
#pragma unroll 4
        for (int i = 0; i < C; ++i) {
          const float o0 = dOc[i * LJ + jj], o1 = dOc[i * LJ + jj + 1];
          const float r0 = dR[i * LJ + jj], r1 = dR[i * LJ + jj + 1];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float qv = Qc[i * LK + kq + KQ * e], kv = Kc[i * LK + kq + KQ * e];
            acc[e][0] = fmaf(qv, o0, fmaf(kv, r0, acc[e][0]));
            acc[e][1] = fmaf(qv, o1, fmaf(kv, r1, acc[e][1]));
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          dS[(kq + KQ * e) * LJ + jj] = acc[e][0];
          dS[(kq + KQ * e) * LJ + jj + 1] = acc[e][1];
        }
      }
    }
  }
  __syncthreads();
  for (int idx = tid; idx < DK * JB; idx += NT) {
    const int kk = idx / JB, j = idx % JB;
    p.dS0[((size_t)bh * DK + kk) * DV + j0 + j] = dS[kk * LJ + j];
  }
}

}  // namespace

template <int DK, int DV>
cudaError_t launch_delta_bwd_typed(const DeltaBwdArgs& args, cudaStream_t stream) {
  constexpr int JB = DV < kJB ? DV : kJB;
  const dim3 grid(args.BH, DV / JB);
  if (args.gains != nullptr) {
    const size_t smem = BwdSmem<DK, JB, true>::BYTES;
    cudaError_t e =
        cudaFuncSetAttribute(delta_bwd_kernel<DK, DV, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    delta_bwd_kernel<DK, DV, true><<<grid, kBwdThreads, smem, stream>>>(args);
    return cudaGetLastError();
  }
  const size_t smem = BwdSmem<DK, JB, false>::BYTES;
  cudaError_t e =
      cudaFuncSetAttribute(delta_bwd_kernel<DK, DV, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  delta_bwd_kernel<DK, DV, false><<<grid, kBwdThreads, smem, stream>>>(args);
  return cudaGetLastError();
}

template <int DK>
cudaError_t launch_delta_bwd_dk(int dv, const DeltaBwdArgs& args, cudaStream_t stream) {
  switch (dv) {
    case 16: return launch_delta_bwd_typed<DK, 16>(args, stream);
    case 32: return launch_delta_bwd_typed<DK, 32>(args, stream);
    case 64: return launch_delta_bwd_typed<DK, 64>(args, stream);
    case 128: return launch_delta_bwd_typed<DK, 128>(args, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_delta_bwd(int dk, int dv, const DeltaBwdArgs& args, cudaStream_t stream) {
  if (args.BH <= 0 || args.L <= 0) return cudaSuccess;
  switch (dk) {
    case 16: return launch_delta_bwd_dk<16>(dv, args, stream);
    case 32: return launch_delta_bwd_dk<32>(dv, args, stream);
    case 64: return launch_delta_bwd_dk<64>(dv, args, stream);
    case 128: return launch_delta_bwd_dk<128>(dv, args, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace kdn
