// Warp-specialised chunked scan for d_k = d_v = 64 or 128 on the sm_100a tensor cores.
//
// The chunk algebra is the generalised WY / UT form of the token recurrence
// S_t = a_t S_{t-1} + g_t e_t^T, e_t = v_t - a_t S_{t-1}^T k_t (A Hippocampus for
// Linear Attention, section 3.3 Eq. (5) and section 3.5; Kalman Delta Networks,
// Abstract, for the Kalman gains): with A_i = prod_{m<=i} a_m and Gam_ij = A_i / A_j,
//
//   (I + N) E = R,   N = strict_lower((K G^T) o Gam),   R = V - diag(A) K S0,
//   O = diag(A) Q S0 + Attn E,   Attn = (Q G^T) o Gam o lower,   T = (I + N)^-1,  E = T R,
//   S_C = A_C S0 + G^T diag(A_C / A_j) E.
//
// Everything that does not involve the state (gates, diagonal variances, gains,
// N, Attn, T) is the "preparation" of a chunk; what does (S0 products, R, E, O,
// the state update) is its "chain".  The CTA runs two groups of 8 warps at once:
// the preparation group works on chunk c + 1 while the chain group works on
// chunk c, so the serial part of each chunk is the chain alone.
//
// The chain runs transposed, with the d_v index on the TMEM lanes, so that every
// state-dependent operand lives in tensor memory and enters the products as the
// A operand (fp16 pairs, one MMA per product):
//
//   D2^T = S0^T [K; Q]^T         A = S0^T (TMEM)      B = [K; Q] tile    -> (K S0)^T | (Q S0)^T
//   E^T  = V^T T^T               A = V^T (smem)       B = T               -> issued before D2 is read
//        - (K S0)^T (T D_A)^T    A = (K S0)^T (TMEM)  B = -T diag(A)      -> E^T (the innovations)
//   (Attn E)^T = E^T Attn^T      A = E^T (TMEM)       B = Attn            -> O = diag(A) (Q S0) + Attn E
//   S_C^T = A_C S0^T + E'^T G    A = E'^T (TMEM)      B = G (or K)        accumulated onto the fp32 master
//
// so the residual R = V - diag(A) K S0 is never formed: its V part runs on the tensor cores while the
// chain converts (K S0)^T, and the decay enters through the preparation's scaled copy of T.  The read-out
// uses Attn E (= AT R, with Attn = lower((Q G^T) o Gam)), so the preparation never forms AT; its one
// product is the row-major [K; Q] G^T.
// fp32 state master and accumulators in TMEM.  Every tensor-core operand is fp16: K and Q are
// converted from bf16 in shared memory when their tile lands (exact in fp16's normal range), the fp32
// operands (state, (K S0), innovations, gains in the state product, T, Attn) are rounded to fp16 once.  A
// float64 emulation of these roundings over 8192-token layers stays below 6e-4 normwise against the exact
// scan, inside the 3e-3 budget for bf16 inputs, while it halves the tensor work and the conversions of the
// bf16 hi/lo form.  The Kalman gains enter [K; Q] G^T as an fp16 hi/lo pair (two products): a read-out
// q_t . g_s that nearly cancels would otherwise carry the gain's rounding relative to |q| |g| (a 2 %
// error on one single-token head at d = 64); with the pair, Attn and N are rounded relative to themselves.
// For the delta-like variants G = K, exact in fp16.
#include <cuda.h>

#include "chunk.h"
#include "chunk_common.cuh"
#include "common.cuh"
#include "mobius.cuh"
#include "sm100.cuh"

namespace kdn {

namespace {

using chunk::kC;
using chunk::kWaitCycles;
using chunk::named_sync;
using chunk::named_sync_or;
using chunk::oct_sum;
using chunk::load8_f16;
using chunk::store8_f16;
using chunk::tok_pair_col;

enum Var : int { kDelta = 0, kDiag = 1, kFull = 2, kIso = 3 };

// Gains of the form beta_t k_t (the delta rule, and the isotropic Kalman filter whose beta_t the
// preparation computes from its one uncertainty scalar per head).
constexpr bool delta_like(int var) { return var == kDelta || var == kIso; }

constexpr int D = 128;
constexpr int NP = D / 64;                 // 64-wide panels across d
constexpr int kThreads = 512;
constexpr int kGroup = 256;                // threads per group; group 0 = chain, group 1 = preparation
constexpr int kBarChain = 1, kBarPrep = 2;  // named barriers of the two groups (0 is __syncthreads)
constexpr int kGD = D / 8;                 // coordinates per thread in the per-token reductions

template <int VAR>
struct WsLayout {
  static constexpr int KQ_PANEL = 128 * 128;             // [K; Q]: 128 rows x 64 (bf16 as loaded, then fp16)
  static constexpr int KQ_BYTES = NP * KQ_PANEL;
  static constexpr int NKQ = delta_like(VAR) ? 3 : 2;    // [K; Q] tiles in flight
  static constexpr int V_PANEL = 64 * 128;
  static constexpr int V_BYTES = NP * V_PANEL;
  static constexpr int G_PANEL = 64 * 128;
  static constexpr int G_HALF = delta_like(VAR) ? 0 : NP * G_PANEL;  // fp16 gains of one slot: hi, then lo
  static constexpr int TAT_HALF = 128 * 128;             // [T; Attn]: 128 rows x 64 fp16
  static constexpr int SCR_BYTES = 64 * chunk::kLD * 4;  // fp32 [64][68]

  static constexpr int OFF_KQ = 0;
  static constexpr int OFF_V = OFF_KQ + NKQ * KQ_BYTES;
  static constexpr int OFF_G = OFF_V + V_BYTES;          // slot s at 2 s G_HALF: fp32 gains, then their fp16 hi | lo
  static constexpr int OFF_TAT = OFF_G + 4 * G_HALF;     // [T; Attn]
  static constexpr int OFF_TAD = OFF_TAT + TAT_HALF;     // -T diag(A) (rows 0..63 used)
  static constexpr int OFF_NF = OFF_TAD + TAT_HALF;
  static constexpr int OFF_TF = OFF_NF + SCR_BYTES;
  static constexpr int TOTAL = OFF_TF + SCR_BYTES;
  static constexpr int SMEM = TOTAL + 1024;              // + alignment slack
  static_assert(delta_like(VAR) || 64 * D * 4 == 2 * G_HALF, "a gain slot holds the fp32 gains before their fp16 copy");
  static_assert(TOTAL <= 216 * 1024, "shared memory budget");

  // TMEM columns
  static constexpr uint32_t T_SM = 0;    // fp32 S^T master: lane j (d_v), column i (d_k)
  static constexpr uint32_t T_SA = 128;  // S0^T as fp16 pairs
  static constexpr uint32_t T_E = 192;   // E^T
  static constexpr uint32_t T_D2 = 256;  // 0..63: (K S0)^T, then its fp16 pairs, then E'^T pairs; 64..127: (Q S0)^T
  static constexpr uint32_t T_AR = 384;  // (Attn E)^T
  static constexpr uint32_t T_D1 = 448;  // [K; Q] G^T (preparation)
  static constexpr uint32_t TMEM_COLS = 512;
};

struct Params {
  const float* beta;
  const float* a;
  const float* r;
  const float* qn;
  float qn_scalar;
  const float* gains;  // full Kalman: [BH, L, D] fp32
  float* S;            // [BH, DT, s_cols]
  int s_cols;          // DT, or 2 DT = 128 at DT = 64: the state [S | M] whose extra columns see zero values
  float* p;            // diag: [BH, D]; isotropic: the uncertainty scalar c, [BH]
  void* o;             // or nullptr
  float* m;
  int out_dtype;
  int L;
  unsigned* status;
};

// Position of coordinate i in a row of the fp32 gain scratch: within each 64-wide block,
// (i % 64) = 8 p + 4 h + e -> 32 h + 4 (p ^ 4 h) + e, so that 32 consecutive coordinates and the
// quads h of chunks p = 0..7 each fall on 32 distinct banks.
__device__ __forceinline__ int gf_pos(int i) {
  const int h = (i >> 2) & 1;
  return (i & ~63) | (h << 5) | ((((i >> 3) & 7) ^ (h << 2)) << 2) | (i & 3);
}

// DT: the head size d_k = d_v (64 or 128).  The tiles and tensor-memory columns are laid out for 128; with
// DT = 64 the upper 64-wide panels of K, Q and V are zero in shared memory (the products over d_k take
// half the K steps, the state product half the columns), the d_v lanes 64..127 carry zeros through the
// chain, and only the true coordinates are read from and written to memory.
template <int VAR, int DT>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_scan_ws_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, Params P) {
  using Lay = WsLayout<VAR>;
  constexpr int NKQ = Lay::NKQ;
  static_assert(DT == 64 || DT == D, "head sizes 64 and 128");
  constexpr int NPT = DT / 64;   // 64-wide panels that hold data
  constexpr int kGDT = DT / 8;   // true coordinates per thread in the per-token reductions
  // The diagonal variant's chain runs the gates and variances of chunk c + 1 while it waits for the
  // preparation of chunk c; the other variants' preparation runs its own gates.
  constexpr bool kChainGates = VAR == kDiag;
  // Who converts each [K; Q] tile from bf16 to fp16 in place: the preparation group for the Kalman
  // variants, whose chain is the longer group; for the delta-like ones the chain, one chunk ahead.
  constexpr bool kConvInPrep = !delta_like(VAR);
  // The diagonal variant's preparation writes Attn after its inverse (see the preparation group)
  constexpr bool kLateAttn = VAR == kDiag;
  constexpr int LD = chunk::kLD;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Vs = sm + Lay::OFF_V;
  uint8_t* TAThi = sm + Lay::OFF_TAT;  // [T; Attn] as fp16
  uint8_t* TADs = sm + Lay::OFF_TAD;   // -T diag(A) as fp16 (rows 0..63)
  float* Nf = reinterpret_cast<float*>(sm + Lay::OFF_NF);
  float* Tf = reinterpret_cast<float*>(sm + Lay::OFF_TF);

  // per-chunk scalars, two slots (chunk c uses slot c & 1)
  __shared__ float sA[2][kC], sB[2][kC], sQ[2][kC];         // a, beta | r, Qn
  __shared__ __align__(16) float4 sVk[VAR == kDiag ? 2 : 1][kC];  // diagonal: (a^2, Qn, 1 / r) per token
  __shared__ float ell[2][kC], gn[2][kC];
  __shared__ __align__(16) float Aex[2][kC];                // A_t
  __shared__ __align__(16) float gcol[2][kC];               // 1 / A_t (times beta_t for the delta rule), when
                                                            // the chunk's decay stays above exp(-80)
  __shared__ __align__(16) float esc[2][kC];                // scale of row t of E in the state update:
                                                            // A_C / A_t (times beta_t for the delta rule)
  __shared__ float en[4][kC];                               // ||e_t||^2 partials per lane quarter
  __shared__ float knorm[kC];                               // isotropic: ||k_t||^2 of the chunk
  __shared__ uint64_t kq_full[NKQ], kq_conv[NKQ], v_full, bar_c, bar_o, bar_p, tat_free;
  __shared__ uint64_t gates_ready[2], prep_done[2], chain_done[2], var_done[2];
  __shared__ uint32_t tmem_base;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int qw = warp & 3;                   // TMEM lane quarter of this warp
  const int gw = (warp & 7);                 // warp within its group
  const int half = gw >> 2;                  // 0 / 1: which half of the columns this thread takes
  const int row = 32 * qw + lane;            // TMEM lane
  const uint32_t t_lane = static_cast<uint32_t>(32 * qw) << 16;
  const int bh = blockIdx.x;
  const int L = P.L;
  const int nchunks = (L + kC - 1) / kC;

  auto issue_kq = [&](int cc) {
    const int slot = cc % NKQ;
    uint8_t* dst = sm + Lay::OFF_KQ + slot * Lay::KQ_BYTES;
    sm100::mbar_arrive_expect_tx(&kq_full[slot], 2 * NPT * 64 * 128);
#pragma unroll
    for (int pn = 0; pn < NPT; ++pn) {
      sm100::tma_load_3d(dst + pn * Lay::KQ_PANEL, &tm_k, &kq_full[slot], 64 * pn, cc * kC, bh);
      sm100::tma_load_3d(dst + pn * Lay::KQ_PANEL + 64 * 128, &tm_q, &kq_full[slot], 64 * pn, cc * kC, bh);
    }
  };
  // bf16 -> fp16 in place over a [K; Q] slot (2 tensors x NPT panels x 64 rows x 8 chunks of 16 bytes) by the
  // 256 threads u of one group, made visible to the tensor cores by the fence
  auto convert_kq = [&](int cc, int u) {
    uint8_t* KQs = sm + Lay::OFF_KQ + (cc % NKQ) * Lay::KQ_BYTES;
#pragma unroll
    for (int r = 0; r < 4 * NPT; ++r) {
      uint4* p4 = reinterpret_cast<uint4*>(KQs) + u + kGroup * r;
      uint4 w = *p4;
      w.x = sm100::bf16x2_to_f16x2(w.x), w.y = sm100::bf16x2_to_f16x2(w.y);
      w.z = sm100::bf16x2_to_f16x2(w.z), w.w = sm100::bf16x2_to_f16x2(w.w);
      *p4 = w;
    }
    sm100::fence_async_smem();
  };
  auto issue_v = [&](int cc) {
    sm100::mbar_arrive_expect_tx(&v_full, NPT * 64 * 128);
#pragma unroll
    for (int pn = 0; pn < NPT; ++pn) sm100::tma_load_3d(Vs + pn * Lay::V_PANEL, &tm_v, &v_full, 64 * pn, cc * kC, bh);
  };

  if (tid == 0) {
    sm100::prefetch_tmap(&tm_q);
    sm100::prefetch_tmap(&tm_k);
    sm100::prefetch_tmap(&tm_v);
#pragma unroll
    for (int i = 0; i < NKQ; ++i) sm100::mbar_init(&kq_full[i], 1), sm100::mbar_init(&kq_conv[i], 1);
    sm100::mbar_init(&v_full, 1);
    sm100::mbar_init(&bar_c, 1);
    sm100::mbar_init(&bar_o, 1);
    sm100::mbar_init(&bar_p, 1);
    sm100::mbar_init(&tat_free, 1);
    for (int i = 0; i < 2; ++i) {
      sm100::mbar_init(&gates_ready[i], 1);
      sm100::mbar_init(&var_done[i], 1);
      sm100::mbar_init(&prep_done[i], 1);
      sm100::mbar_init(&chain_done[i], 1);
    }
    sm100::fence_mbar_init();
    for (int cc = 0; cc < NKQ && cc < nchunks; ++cc) issue_kq(cc);
    issue_v(0);
  }
  if (DT < D) {  // the upper panels of every [K; Q] slot and of V: zero for the whole launch
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (int e = tid; e < NKQ * 1024; e += kThreads)
      reinterpret_cast<uint4*>(sm + Lay::OFF_KQ + (e / 1024) * Lay::KQ_BYTES + Lay::KQ_PANEL)[e % 1024] = z;
    for (int e = tid; e < 512; e += kThreads) reinterpret_cast<uint4*>(Vs + Lay::V_PANEL)[e] = z;
    sm100::fence_async_smem();
  }
  if (warp == 0) {
    sm100::tmem_alloc(&tmem_base, Lay::TMEM_COLS);
    sm100::tmem_relinquish();
  }
  // raw per-token scalars of chunk cc into registers (threads 0..63 of the preparation group); chunk 0's
  // go to slot 0 before the groups part, chunk c + 1's are stored by the preparation of chunk c
  float ra = 1.f, rb = 0.f, rq = 0.f;
  auto fetch_scalars = [&](int cc) {
    const int u = tid - kGroup;
    if (u >= 0 && u < kC) {
      const int tok = cc * kC + u;
      const bool valid = tok < L;
      const size_t ti = (size_t)bh * L + tok;
      ra = valid ? (P.a ? P.a[ti] : 1.f) : 1.f;
      if (VAR == kDelta) rb = valid ? P.beta[ti] : 0.f;
      else rb = valid ? P.r[ti] : 1.f;
      rq = valid ? (P.qn ? P.qn[ti] : P.qn_scalar) : 0.f;
    }
  };
  auto store_scalars = [&](int slot) {
    const int u = tid - kGroup;
    if (u >= 0 && u < kC) {
      sA[slot][u] = ra, sB[slot][u] = rb, sQ[slot][u] = rq;
      if (VAR == kDiag) sVk[slot][u] = make_float4(ra * ra, rq, 1.f / rb, 0.f);
    }
  };
  // gates of chunk cc into its slot, by one warp: inclusive prefix sums of log a over the chunk (a gate of 0
  // enters as exp(-60)), A_t, and the state-update row scale A_C / A_t (times beta_t for the delta rule)
  auto run_gates = [&](int cc) {
    const int sl = cc & 1;
    float x0 = sA[sl][lane], x1 = sA[sl][32 + lane];
    x0 = x0 > 0.f ? fmaxf(__logf(x0), -60.f) : -60.f;
    x1 = x1 > 0.f ? fmaxf(__logf(x1), -60.f) : -60.f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y0 = __shfl_up_sync(0xffffffffu, x0, o), y1 = __shfl_up_sync(0xffffffffu, x1, o);
      if (lane >= o) x0 += y0, x1 += y1;
    }
    x1 += __shfl_sync(0xffffffffu, x0, 31);
    const float lC = __shfl_sync(0xffffffffu, x1, 31);
    ell[sl][lane] = x0, ell[sl][32 + lane] = x1;
    Aex[sl][lane] = __expf(x0), Aex[sl][32 + lane] = __expf(x1);
    const float r0 = __expf(lC - x0), r1 = __expf(lC - x1);  // A_C / A_t without a division
    esc[sl][lane] = delta_like(VAR) ? r0 * sB[sl][lane] : r0;
    esc[sl][32 + lane] = delta_like(VAR) ? r1 * sB[sl][32 + lane] : r1;
    // Gam_ij = A_i (1 / A_j) without an exponential per pair: safe (no overflow) while ell_C >= -80
    gcol[sl][lane] = __expf(-x0) * (delta_like(VAR) ? sB[sl][lane] : 1.f);
    gcol[sl][32 + lane] = __expf(-x1) * (delta_like(VAR) ? sB[sl][32 + lane] : 1.f);
  };
  fetch_scalars(0);
  store_scalars(0);
  if (nchunks > 1) fetch_scalars(1);
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = tmem_base;

  // Diagonal variances of chunk cc (independent of v and S), run by the chain one chunk ahead, in its wait
  // for the preparation.  Per coordinate: p^- = a^2 p + Qn, pk = p^- k, p <- p^- r / (r + pk k), on the
  // homogeneous pair p = x / y: token t maps (x, y) by [[a^2, Qn], [w a^2, w Qn + 1]] (w = k^2 / r; the
  // token's map [[r a^2, r Qn], [k^2 a^2, k^2 Qn + r]] divided by r), i.e. x' = a^2 x + Qn y = p^- y and
  // y' = y + w x': a multiply and two multiply-adds of serial chain per token; the divisions that recover
  // the gains p^- k = x' k / y are batched after each four tokens' steps (in-order issue would otherwise
  // hold the chain behind every reciprocal), and a power-of-two rescale every eight tokens is exact
  // (x / y does not change).  One thread per coordinate steps
  // all 64 tokens: this phase issues beside the preparation group, and a split of the tokens over threads
  // (composing the earlier tokens' maps) only adds instructions, while the direct form p <- r p^- / s puts
  // a division on the serial chain.  The unnormalised gains pk go, fp32, into the gain slot of chunk cc;
  // p after the chunk stays in the thread.
  auto run_variances = [&](int cc, int i, float& pcur) {
    if (VAR == kDiag) {
      const int sl = cc & 1;
      // keys from the chunk's K tile as it landed (bf16): the preparation converts that tile to fp16 only
      // after these variances are done
      const uint8_t* Kp = sm + Lay::OFF_KQ + (cc % NKQ) * Lay::KQ_BYTES + (i / 64) * Lay::KQ_PANEL;
      float* Gw = reinterpret_cast<float*>(sm + Lay::OFF_G + 2 * sl * Lay::G_HALF);
      const int gpos = gf_pos(i);
      float x = pcur, y = 1.f;
      // keys and (a^2, Qn, 1 / r) of four tokens into registers a group ahead of their use
      auto load4 = [&](int t4, float (&kq)[4], float4 (&sq)[4]) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          kq[u] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(Kp + sm100::sw128(t4 + u, i % 64)));
          sq[u] = sVk[sl][t4 + u];
        }
      };
      // the serial part of four tokens (two multiply-adds and a multiply each), then their gains: the
      // reciprocals and stores issue after the chain steps, not between them
      auto step4 = [&](int t4, const float (&kq)[4], const float4 (&sq)[4]) {
        float num[4], den[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float xm = fmaf(sq[u].x, x, sq[u].y * y);
          num[u] = xm * kq[u], den[u] = y;
          x = xm;
          y = fmaf(kq[u] * kq[u] * sq[u].z, xm, y);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) Gw[(t4 + u) * D + gpos] = __fdividef(num[u], den[u]);
      };
      float ka[4], kb[4];
      float4 va[4], vb[4];
      load4(0, ka, va);
#pragma unroll 1
      for (int t8 = 0; t8 < kC; t8 += 8) {
        load4(t8 + 4, kb, vb);
        step4(t8, ka, va);
        load4((t8 + 8) & (kC - 1), ka, va);  // (the last one reloads tokens 0..3, unused)
        step4(t8 + 4, kb, vb);
        const int ey = min((__float_as_int(y) >> 23) & 0xff, 253);
        const float sc = __int_as_float((254 - ey) << 23);  // 2^(127 - ey), exact
        x *= sc, y *= sc;
      }
      pcur = __fdividef(x, y);
    }
  };

  if (tid < kGroup) {
    // =============================================================================== chain group
    const int j = row;                       // d_v index
    const bool leader = tid == 0;            // issues the chain's products and every TMA load
    bool aborted = false;
    uint32_t ph_c = 0, ph_o = 0;
    auto gwait = [&](uint64_t* b, uint32_t parity) -> bool {
      bool bad = false;
      if (leader) bad = !sm100::mbar_wait_bounded(b, parity, kWaitCycles);
      bad = named_sync_or(kBarChain, kGroup, bad);
      if (bad && leader) raise_status(P.status, kStatusTimeout);
      sm100::tc_fence_after();
      return !bad;
    };
    // S0^T pairs for the next [K; Q] product and the master pre-scaled by the next chunk's A_C:
    // x = S[64 half + 32 v .. + 31][j]
    // x = S[dk0 .. dk0 + 31][j]
    auto emit_state = [&](float (&x)[32], int dk0, float scale) {
      float hw[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) hw[e] = __uint_as_float(sm100::pack2_f16(x[2 * e], x[2 * e + 1]));
      sm100::tmem_st16(tmem + t_lane + Lay::T_SA + dk0 / 2, hw);
#pragma unroll
      for (int e = 0; e < 32; ++e) x[e] *= scale;
      sm100::tmem_st32(tmem + t_lane + Lay::T_SM + dk0, x);
    };
    // D2^T = S0^T [K; Q]^T, K steps 4 part .. 4 part + 3 (d_k 64 part ..): issued as soon as that half of
    // the S0^T pairs is in tensor memory; the second half commits
    auto issue_d2 = [&](uint32_t kq_addr, int part) {
      constexpr uint32_t id = sm100::idesc_f16(128, 128, false, false);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int ks = 4 * part + u;
        const uint64_t b = sm100::smem_desc(kq_addr + (ks / 4) * Lay::KQ_PANEL + (ks % 4) * 32, 16, 1024);
        sm100::mma_bf16_ts(tmem + Lay::T_D2, tmem + Lay::T_SA + 8 * ks, b, id, ks > 0);
      }
      if (part == NPT - 1) sm100::mma_commit(&bar_c);
    };
    auto kq_addr_of = [&](int cc) { return sm100::smem_u32(sm + Lay::OFF_KQ + (cc % NKQ) * Lay::KQ_BYTES); };

    // diagonal: p of coordinate tid (threads 0..D-1, warps 0..3, run the variances; warp 4 the gates)
    const bool var_thread = VAR == kDiag && tid < DT;
    float pcur = var_thread ? P.p[(size_t)bh * DT + tid] : 1.f;
    const int SC = P.s_cols;
    float* Sg = P.S + (size_t)bh * DT * SC;
    if (!kConvInPrep) {  // [K; Q] of chunk 0
      if (!gwait(&kq_full[0], 0)) {
        aborted = true;
      } else {
        convert_kq(0, tid);
        named_sync(kBarChain, kGroup);
        if (leader) sm100::mbar_arrive(&kq_conv[0]);
      }
    }
    if (!aborted && kChainGates) {  // gates and variances of chunk 0 (its scalars are in slot 0 already)
      if (!gwait(&kq_full[0], 0)) {
        aborted = true;
      } else {
        if (var_thread) run_variances(0, tid, pcur);
        if (gw == 4) run_gates(0);
        named_sync(kBarChain, kGroup);
        if (leader) sm100::mbar_arrive(&var_done[0]);
      }
    }
    if (aborted || (!kChainGates && !gwait(&gates_ready[0], 0)) || !gwait(&kq_conv[0], 0)) {
      aborted = true;
    } else {
      const float AC0 = Aex[0][kC - 1];
#pragma unroll
      for (int v = 0; v < NPT; ++v) {
        float x[32];
        const int dk0 = 32 * half + 64 * v;
#pragma unroll
        for (int u = 0; u < 32; ++u) x[u] = (DT == D || j < SC) ? Sg[(size_t)(dk0 + u) * SC + j] : 0.f;
        emit_state(x, dk0, AC0);
        sm100::tmem_wait_st();
        sm100::tc_fence_before();
        named_sync(kBarChain, kGroup);
        sm100::tc_fence_after();
        if (leader) issue_d2(kq_addr_of(0), v);
      }
    }

    const uint32_t tat_hi = sm100::smem_u32(TAThi);
    for (int c = 0; c < nchunks && !aborted; ++c) {
      const int s = c & 1, kslot = c % NKQ;
      const int t0 = c * kC;
      const uint32_t kq0 = sm100::smem_u32(sm + Lay::OFF_KQ + kslot * Lay::KQ_BYTES);

      // D2^T = S0^T [K; Q]^T of this chunk was issued with its state operands (end of the previous chunk)

      // ---------------------------------------------------------------- V of this chunk to fp16, the gates
      {
        bool bad = false;
        if (leader) {
          bad = !sm100::mbar_wait_bounded(&v_full, c & 1, kWaitCycles) ||
                !sm100::mbar_wait_bounded(&gates_ready[s], (c >> 1) & 1, kWaitCycles);
          if (!bad && (!kConvInPrep || kChainGates) && c + 1 < nchunks)
            bad = !sm100::mbar_wait_bounded(&kq_full[(c + 1) % NKQ], ((c + 1) / NKQ) & 1, kWaitCycles);
        }
        bad = named_sync_or(kBarChain, kGroup, bad);
        if (bad) {
          if (leader) raise_status(P.status, kStatusTimeout);
          aborted = true;
          break;
        }
        // NPT panels x 64 rows x 8 chunks of 16 bytes, in place (made visible to the MMA by the fence here and
        // the barrier below): the diagonal variant's warps 4..7 convert while warps 0..3 step the variances of
        // chunk c + 1 and warp 4 runs its gates (its scalars were stored before gates_ready of chunk c; its keys
        // are read before the preparation converts their tile, which waits for var_done)
        constexpr int kConvThreads = kChainGates ? kGroup / 2 : kGroup;
        const int cv = kChainGates ? tid - kGroup / 2 : tid;
        if (cv >= 0) {
#pragma unroll
          for (int u = 0; u < 2 * NPT * kGroup / kConvThreads; ++u) {
            uint4* p4 = reinterpret_cast<uint4*>(Vs) + cv + kConvThreads * u;
            uint4 w = *p4;
            w.x = sm100::bf16x2_to_f16x2(w.x), w.y = sm100::bf16x2_to_f16x2(w.y);
            w.z = sm100::bf16x2_to_f16x2(w.z), w.w = sm100::bf16x2_to_f16x2(w.w);
            *p4 = w;
          }
          sm100::fence_async_smem();
        }
        if (kChainGates) {
          if (c + 1 < nchunks) {
            if (var_thread) run_variances(c + 1, tid, pcur);
            if (gw == 4) run_gates(c + 1);
          }
          named_sync(kBarChain, kGroup);
          if (leader && c + 1 < nchunks) sm100::mbar_arrive(&var_done[(c + 1) & 1]);
        } else if (!kConvInPrep && c + 1 < nchunks) {  // [K; Q] of the next chunk, for the preparation
          convert_kq(c + 1, tid);
          named_sync(kBarChain, kGroup);
          if (leader) sm100::mbar_arrive(&kq_conv[(c + 1) % NKQ]);
        }
      }

      // ---------------------------------------------------------------- E^T = V^T T^T, queued behind the S0 product
      if (!gwait(&prep_done[s], (c >> 1) & 1)) { aborted = true; break; }
      if (leader) {
        constexpr uint32_t id = sm100::idesc_f16(128, 64, true, false);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t a = sm100::smem_desc(sm100::smem_u32(Vs) + ks * 2048, Lay::V_PANEL, 1024);
          sm100::mma_bf16(tmem + Lay::T_E, a, sm100::smem_desc(tat_hi + ks * 32, 16, 1024), id, ks > 0);
        }
      }

      // ---------------------------------------------------------------- (K S0)^T to fp16 pairs, in place
      {
        if (!gwait(&bar_c, ph_c)) { aborted = true; break; }
        ph_c ^= 1;
        // without the delta rule the state product reads G, not K: this slot's K, Q are dead once the S0
        // product is (the preparation was done with them before prep_done), so the tile two chunks ahead
        // loads a whole chain phase earlier than at the chunk's end
        if (!delta_like(VAR) && leader && c + NKQ < nchunks) issue_kq(c + NKQ);
        float X[32];
        sm100::tmem_ld32(tmem + t_lane + Lay::T_D2 + 32 * half, X);
        sm100::tmem_wait_ld();
        float hw[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) hw[e] = __uint_as_float(sm100::pack2_f16(X[2 * e], X[2 * e + 1]));
        sm100::tmem_st16(tmem + t_lane + Lay::T_D2 + 32 * half, hw);
        sm100::tmem_wait_st();
      }
      sm100::tc_fence_before();
      named_sync(kBarChain, kGroup);
      sm100::tc_fence_after();

      // ---------------------------------------------------------------- E^T -= (K S0)^T (T diag(A))^T
      if (leader) {
        constexpr uint32_t id = sm100::idesc_f16(128, 64, false, false);
        const uint32_t tad = sm100::smem_u32(TADs);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t a = tmem + Lay::T_D2 + tok_pair_col(ks);
          sm100::mma_bf16_ts(tmem + Lay::T_E, a, sm100::smem_desc(tad + ks * 32, 16, 1024), id, true);
        }
        sm100::mma_commit(&bar_c);
      }
      if (!gwait(&bar_c, ph_c)) { aborted = true; break; }
      ph_c ^= 1;
      if (leader && c + 1 < nchunks) issue_v(c + 1);  // V of this chunk is dead

      // ---------------------------------------------------------------- E' pairs; S^T master += E'^T G; ||e||^2
      float E[32];
      {
        sm100::tmem_ld32(tmem + t_lane + Lay::T_E + 32 * half, E);
        sm100::tmem_wait_ld();
        const float4* S4 = reinterpret_cast<const float4*>(&esc[s][32 * half]);
        float hw[16], ew[16];
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 sv = S4[e4];
          hw[2 * e4] = __uint_as_float(sm100::pack2_f16(E[4 * e4] * sv.x, E[4 * e4 + 1] * sv.y));
          hw[2 * e4 + 1] = __uint_as_float(sm100::pack2_f16(E[4 * e4 + 2] * sv.z, E[4 * e4 + 3] * sv.w));
          ew[2 * e4] = __uint_as_float(sm100::pack2_f16(E[4 * e4], E[4 * e4 + 1]));
          ew[2 * e4 + 1] = __uint_as_float(sm100::pack2_f16(E[4 * e4 + 2], E[4 * e4 + 3]));
        }
        sm100::tmem_st16(tmem + t_lane + Lay::T_D2 + 32 * half, hw);  // E' pairs, over the dead (K S0) pairs
        sm100::tmem_st16(tmem + t_lane + Lay::T_E + 32 * half, ew);   // E pairs, in place
      }
      sm100::tmem_wait_st();
      sm100::tc_fence_before();
      named_sync(kBarChain, kGroup);
      sm100::tc_fence_after();
      if (leader) {
        // (Attn E)^T = E^T Attn^T for the read-out first (it frees [T; Attn]), then the state product
        constexpr uint32_t ido = sm100::idesc_f16(128, 64, false, false);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          sm100::mma_bf16_ts(tmem + Lay::T_AR, tmem + Lay::T_E + tok_pair_col(ks),
                             sm100::smem_desc(tat_hi + 64 * 128 + ks * 32, 16, 1024), ido, ks > 0);
        sm100::mma_commit(&bar_o);
        sm100::mma_commit(&tat_free);
        constexpr uint32_t id = sm100::idesc_f16(128, DT, false, true);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t ah = tmem + Lay::T_D2 + tok_pair_col(ks);
          if (delta_like(VAR)) {
            const uint64_t bk = sm100::smem_desc(kq0 + ks * 2048, Lay::KQ_PANEL, 1024);
            sm100::mma_bf16_ts(tmem + Lay::T_SM, ah, bk, id, true);
          } else {
            const uint32_t g0 = sm100::smem_u32(sm + Lay::OFF_G + 2 * s * Lay::G_HALF);
            const uint64_t bgh = sm100::smem_desc(g0 + ks * 2048, Lay::G_PANEL, 1024);
            sm100::mma_bf16_ts(tmem + Lay::T_SM, ah, bgh, id, true);
          }
        }
        sm100::mma_commit(&bar_c);
      }
      // sum of E^2 over this warp's 32 lanes for each of the 32 tokens, while the state product runs: after
      // the butterfly lane l holds token 32 half + l
#pragma unroll
      for (int u = 0; u < 32; ++u) E[u] *= E[u];
#pragma unroll
      for (int k = 16; k >= 1; k >>= 1) {
        const bool up = (lane & k) != 0;
#pragma unroll
        for (int i = 0; i < k; ++i) {
          const float send = up ? E[i] : E[i + k];
          const float keep = up ? E[i + k] : E[i];
          E[i] = keep + __shfl_xor_sync(0xffffffffu, send, k);
        }
      }
      en[qw][32 * half + lane] = E[0];
      // O = diag(A) Q S0 + Attn E (Attn E = AT R), while the state product runs (it touches neither column range)
      if (!gwait(&bar_o, ph_o)) { aborted = true; break; }
      ph_o ^= 1;
      {
        const bool full = t0 + kC <= L;
        const float4* A4 = reinterpret_cast<const float4*>(&Aex[s][32 * half]);
        const size_t base = ((size_t)bh * L + t0 + 32 * half) * DT + j;
        const bool own = (DT == D || j < DT) && P.o != nullptr;  // a true d_v coordinate (warp-uniform)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float Y[16], Oi[16];
          sm100::tmem_ld16(tmem + t_lane + Lay::T_D2 + 64 + 32 * half + 16 * hh, Y);
          sm100::tmem_ld16(tmem + t_lane + Lay::T_AR + 32 * half + 16 * hh, Oi);
          sm100::tmem_wait_ld();
          float ov[16];
#pragma unroll
          for (int u4 = 0; u4 < 4; ++u4) {
            const float4 av = A4[4 * hh + u4];
            ov[4 * u4] = fmaf(av.x, Y[4 * u4], Oi[4 * u4]);
            ov[4 * u4 + 1] = fmaf(av.y, Y[4 * u4 + 1], Oi[4 * u4 + 1]);
            ov[4 * u4 + 2] = fmaf(av.z, Y[4 * u4 + 2], Oi[4 * u4 + 2]);
            ov[4 * u4 + 3] = fmaf(av.w, Y[4 * u4 + 3], Oi[4 * u4 + 3]);
          }
          if (!own) {
          } else if (P.out_dtype == kF32) {
            float* op = reinterpret_cast<float*>(P.o) + base + (size_t)(16 * hh) * DT;
#pragma unroll
            for (int u = 0; u < 16; ++u)
              if (full || t0 + 32 * half + 16 * hh + u < L) op[u * DT] = ov[u];
          } else {
            __nv_bfloat16* op = reinterpret_cast<__nv_bfloat16*>(P.o) + base + (size_t)(16 * hh) * DT;
#pragma unroll
            for (int u = 0; u < 16; ++u)
              if (full || t0 + 32 * half + 16 * hh + u < L) op[u * DT] = __float2bfloat16_rn(ov[u]);
          }
        }
      }
      if (!gwait(&bar_c, ph_c)) { aborted = true; break; }  // also: every lane quarter's norms are in
      ph_c ^= 1;
      if (tid < kC && P.m != nullptr && t0 + tid < L)
        P.m[(size_t)bh * L + t0 + tid] = sqrtf(gn[s][tid]) * sqrtf(en[0][tid] + en[1][tid] + en[2][tid] + en[3][tid]);

      // ---------------------------------------------------------------- state operands of the next chunk, and its
      // S0 product, a half at a time
      if (c + 1 < nchunks) {
        if (!kChainGates && !gwait(&gates_ready[s ^ 1], ((c + 1) >> 1) & 1)) { aborted = true; break; }
        if (!gwait(&kq_conv[(c + 1) % NKQ], ((c + 1) / NKQ) & 1)) { aborted = true; break; }
        const float ACn = Aex[s ^ 1][kC - 1];
        const uint32_t kq_next = kq_addr_of(c + 1);
#pragma unroll
        for (int v = 0; v < NPT; ++v) {
          float x[32];
          const int dk0 = 32 * half + 64 * v;
          sm100::tmem_ld32(tmem + t_lane + Lay::T_SM + dk0, x);
          sm100::tmem_wait_ld();
          emit_state(x, dk0, ACn);
          sm100::tmem_wait_st();
          sm100::tc_fence_before();
          named_sync(kBarChain, kGroup);
          sm100::tc_fence_after();
          if (leader) issue_d2(kq_next, v);
        }
      } else {
        sm100::tc_fence_before();
        named_sync(kBarChain, kGroup);
        sm100::tc_fence_after();
      }
      if (leader) {
        sm100::mbar_arrive(&chain_done[s]);
        if (delta_like(VAR) && c + NKQ < nchunks) issue_kq(c + NKQ);  // this slot's K, Q are dead
      }
    }
    if (!aborted && (DT == D || (half == 0 && j < SC))) {  // warp-uniform: true d_k columns, state lanes
#pragma unroll
      for (int v = 0; v < 2; ++v) {
        float x[32];
        sm100::tmem_ld32(tmem + t_lane + Lay::T_SM + 64 * half + 32 * v, x);
        sm100::tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 32; ++u) Sg[(size_t)(64 * half + 32 * v + u) * SC + j] = x[u];
      }
    }
    if (!aborted && var_thread) P.p[(size_t)bh * DT + tid] = pcur;
  } else {
    // =============================================================================== preparation group
    const int pt = tid - kGroup;
    const bool leader = pt == 0;             // issues the preparation's products
    bool aborted = false;
    uint32_t ph_p = 0;
    float c_iso = VAR == kIso ? P.p[bh] : 0.f;  // isotropic: the uncertainty scalar, carried by the gates warp

    for (int c = 0; c < nchunks; ++c) {
      const int s = c & 1, kslot = c % NKQ;
      const int t0 = c * kC;
      uint8_t* KQ = sm + Lay::OFF_KQ + kslot * Lay::KQ_BYTES;
      const uint32_t kq0 = sm100::smem_u32(KQ);
      uint8_t* Ghi = sm + Lay::OFF_G + 2 * s * Lay::G_HALF;

      // ---------------------------------------------------------------- slot s free (chain of c - 2), K, Q of c
      {
        bool bad = false;
        if (leader) {
          if (c >= 2) bad = !sm100::mbar_wait_bounded(&chain_done[s], ((c - 2) >> 1) & 1, kWaitCycles);
          if (!bad) bad = !sm100::mbar_wait_bounded(kConvInPrep ? &kq_full[kslot] : &kq_conv[kslot], (c / NKQ) & 1,
                                                    kWaitCycles);
        }
        bad = named_sync_or(kBarPrep, kGroup, bad);
        if (bad) {
          if (leader) raise_status(P.status, kStatusTimeout);
          aborted = true;
          break;
        }
      }
      // ---------------------------------------------------------------- K, Q of this chunk: bf16 -> fp16 in place
      // (the diagonal variant's chain reads the bf16 keys for its variances first: converted below)
      if (kConvInPrep && !kChainGates) {
        convert_kq(c, pt);
        named_sync(kBarPrep, kGroup);
        if (leader) sm100::mbar_arrive(&kq_conv[kslot]);
      }
      // ---------------------------------------------------------------- isotropic: beta of this chunk
      if (VAR == kIso) {
        // ||k_t||^2 (eight threads per token, two passes of 32 tokens)
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
          const int t = 32 * pass + (pt >> 3), part = pt & 7;
          float sq = 0.f;
#pragma unroll
          for (int pn = 0; pn < NPT; ++pn) {
            float xk[8];
            load8_f16(KQ + pn * Lay::KQ_PANEL, sm100::sw128_chunk(t, part), xk);
#pragma unroll
            for (int e = 0; e < 8; ++e) sq = fmaf(xk[e], xk[e], sq);
          }
          sq = oct_sum(sq);
          if (part == 0) knorm[t] = sq;
        }
        named_sync(kBarPrep, kGroup);
        if (gw == 4) {
          // The uncertainty scalar's token maps (Kalman Delta Networks, Abstract: Moebius maps, scanned
          // associatively): two tokens per lane, an inclusive scan over the lanes, then each lane steps its
          // two tokens exactly from the carried value and writes beta_t over r_t.
          mobius::Mob mine = mobius::identity();
          float a2[2], qv[2], rv[2], kk[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int t = 2 * lane + u;
            a2[u] = sA[s][t] * sA[s][t], qv[u] = sQ[s][t], rv[u] = sB[s][t], kk[u] = knorm[t];
            mine = mobius::compose(mobius::iso_token(a2[u], qv[u], kk[u] / (DT * rv[u])), mine);
          }
          mobius::Mob incl = mine;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const mobius::Mob left = mobius::shfl_up(incl, o);
            if (lane >= o) incl = mobius::compose(incl, left);
          }
          mobius::Mob excl = mobius::shfl_up(incl, 1);
          if (lane == 0) excl = mobius::identity();
          float cv = mobius::apply(excl, c_iso);
          bool bad = false;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const float cm = fmaf(a2[u], cv, qv[u]);
            const float sden = fmaf(cm, kk[u], rv[u]);
            bad |= !(sden > 0.f && isfinite(sden) && cm >= 0.f);
            sB[s][2 * lane + u] = cm / sden;
            cv = DT * cm * rv[u] / fmaf((float)DT, rv[u], cm * kk[u]);
          }
          if (bad && t0 + 2 * lane < L) raise_status(P.status, kStatusNumeric);
          c_iso = __shfl_sync(0xffffffffu, cv, 31);
          __syncwarp();
        }
      }
      // ---------------------------------------------------------------- gates | diagonal variances
      if (!kChainGates && gw == 4) run_gates(c);
      if (c + 1 < nchunks) {  // raw scalars of the next chunk (its slot was last read by chunk c - 1)
        store_scalars(s ^ 1);
        if (c + 2 < nchunks) fetch_scalars(c + 2);
      }
      named_sync(kBarPrep, kGroup);
      // gates_ready: this chunk's gates (unless the chain runs them) and the next chunk's raw scalars
      if (leader) sm100::mbar_arrive(&gates_ready[s]);
      if (kChainGates) {  // the chain has run this chunk's gates and written its unnormalised gains into slot s
        bool bad = false;
        if (leader) bad = !sm100::mbar_wait_bounded(&var_done[s], (c >> 1) & 1, kWaitCycles);
        bad = named_sync_or(kBarPrep, kGroup, bad);
        if (bad) {
          if (leader) raise_status(P.status, kStatusTimeout);
          aborted = true;
          break;
        }
        convert_kq(c, pt);
        named_sync(kBarPrep, kGroup);
        if (leader) sm100::mbar_arrive(&kq_conv[kslot]);
      }

      // ---------------------------------------------------------------- gains: norms, hi/lo panels (8 threads per token)
      {
        // Thread `part` of token t takes the 16-byte chunk `part` of every 64-wide panel: coordinates
        // 64 pn + 8 part .. + 7, so each group of eight lanes reads and writes one whole 128-byte row.
        // The diagonal variant normalises the fp32 gains that share the slot with their fp16 copy: all
        // of them are read before any of the copy is written.
        const int part = pt & 7;
        float g[2][kGD];
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
          const int t = 32 * pass + (pt >> 3);
          float kv[kGD];
#pragma unroll
          for (int pn = 0; pn < NPT; ++pn) {
            float xk[8];
            load8_f16(KQ + pn * Lay::KQ_PANEL, sm100::sw128_chunk(t, part), xk);
#pragma unroll
            for (int e = 0; e < 8; ++e) kv[8 * pn + e] = xk[e];
          }
          if (delta_like(VAR)) {
            float sq = 0.f;
#pragma unroll
            for (int e = 0; e < kGDT; ++e) sq = fmaf(kv[e], kv[e], sq);
            sq = oct_sum(sq);
            if (part == 0) gn[s][t] = sB[s][t] * sB[s][t] * sq;
          } else {
            if (VAR == kDiag) {
              const float* Gw = reinterpret_cast<const float*>(Ghi);
#pragma unroll
              for (int pn = 0; pn < NPT; ++pn)
#pragma unroll
                for (int hq = 0; hq < 2; ++hq) {
                  const float4 x4 = *reinterpret_cast<const float4*>(Gw + t * D + gf_pos(64 * pn + 8 * part + 4 * hq));
                  g[pass][8 * pn + 4 * hq] = x4.x, g[pass][8 * pn + 4 * hq + 1] = x4.y;
                  g[pass][8 * pn + 4 * hq + 2] = x4.z, g[pass][8 * pn + 4 * hq + 3] = x4.w;
                }
              float sd = 0.f;
#pragma unroll
              for (int e = 0; e < kGDT; ++e) sd = fmaf(g[pass][e], kv[e], sd);
              sd = oct_sum(sd) + sB[s][t];
              if (part == 0 && !(sd > 0.f && isfinite(sd))) raise_status(P.status, kStatusNumeric);
              const float inv_s = 1.f / sd;
#pragma unroll
              for (int e = 0; e < kGDT; ++e) g[pass][e] *= inv_s;
            } else {
              const bool valid = t0 + t < L;
              const float* gp = P.gains + ((size_t)bh * L + t0 + t) * DT + 8 * part;
#pragma unroll
              for (int pn = 0; pn < NPT; ++pn)
#pragma unroll
                for (int hq = 0; hq < 2; ++hq) {
                  float4 x4 = make_float4(0.f, 0.f, 0.f, 0.f);
                  if (valid) x4 = *reinterpret_cast<const float4*>(gp + 64 * pn + 4 * hq);
                  g[pass][8 * pn + 4 * hq] = x4.x, g[pass][8 * pn + 4 * hq + 1] = x4.y;
                  g[pass][8 * pn + 4 * hq + 2] = x4.z, g[pass][8 * pn + 4 * hq + 3] = x4.w;
                }
            }
            float n2 = 0.f;
#pragma unroll
            for (int e = 0; e < kGDT; ++e) n2 = fmaf(g[pass][e], g[pass][e], n2);
            n2 = oct_sum(n2);
            if (part == 0) gn[s][t] = n2;
          }
        }
        if (!delta_like(VAR)) {
          if (VAR == kDiag) named_sync(kBarPrep, kGroup);
#pragma unroll
          for (int pass = 0; pass < 2; ++pass) {
            const int t = 32 * pass + (pt >> 3);
#pragma unroll
            for (int pn = 0; pn < NPT; ++pn) {
              float xg[8], xl[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                xg[e] = g[pass][8 * pn + e];
                xl[e] = xg[e] - __half2float(__float2half_rn(xg[e]));
              }
              store8_f16(Ghi, pn * Lay::G_PANEL + sm100::sw128_chunk(t, part), xg);
              store8_f16(Ghi + Lay::G_HALF, pn * Lay::G_PANEL + sm100::sw128_chunk(t, part), xl);
            }
          }
        }
      }
      sm100::fence_async_smem();
      sm100::tc_fence_before();
      named_sync(kBarPrep, kGroup);
      sm100::tc_fence_after();

      // ---------------------------------------------------------------- D1 = [K; Q] G^T
      if (leader) {
        constexpr uint32_t id1 = sm100::idesc_f16(128, 64, false, false);
        const uint32_t ghi = sm100::smem_u32(Ghi);
#pragma unroll
        for (int ks = 0; ks < DT / 16; ++ks) {
          const uint32_t koff = (ks / 4) * Lay::KQ_PANEL + (ks % 4) * 32;
          const uint64_t a = sm100::smem_desc(kq0 + koff, 16, 1024);
          if (delta_like(VAR)) {
            sm100::mma_bf16(tmem + Lay::T_D1, a, a, id1, ks > 0);  // G = K (beta enters with Gam)
          } else {
            const uint32_t goff = (ks / 4) * Lay::G_PANEL + (ks % 4) * 32;
            sm100::mma_bf16(tmem + Lay::T_D1, a, sm100::smem_desc(ghi + goff, 16, 1024), id1, ks > 0);
            sm100::mma_bf16(tmem + Lay::T_D1, a, sm100::smem_desc(ghi + Lay::G_HALF + goff, 16, 1024), id1, true);
          }
        }
        sm100::mma_commit(&bar_p);
      }
      auto prep_wait = [&](uint64_t* b, uint32_t parity) -> bool {
        bool bad = false;
        if (leader) bad = !sm100::mbar_wait_bounded(b, parity, kWaitCycles);
        bad = named_sync_or(kBarPrep, kGroup, bad);
        if (bad && leader) raise_status(P.status, kStatusTimeout);
        sm100::tc_fence_after();
        return !bad;
      };
      {
        bool bad = false;
        if (leader) {
          bad = !sm100::mbar_wait_bounded(&bar_p, ph_p, kWaitCycles);
          if (!bad && !kLateAttn && c >= 1) bad = !sm100::mbar_wait_bounded(&tat_free, (c - 1) & 1, kWaitCycles);
        }
        bad = named_sync_or(kBarPrep, kGroup, bad);
        if (bad) {
          if (leader) raise_status(P.status, kStatusTimeout);
          aborted = true;
          break;
        }
        sm100::tc_fence_after();
        ph_p ^= 1;
      }

      // Y_ij (beta_j) Gam_ij from the D1 lanes of this warp: as A_i times the column factor when the chunk's
      // decay allows it, else by one exponential per pair (chunks with strong resets); the choice is uniform
      // over the chunk.  N (lanes 0..63) goes to the fp32 scratch, Attn (lanes 64..127) into [T; Attn] once the
      // chain's read-out product of the previous chunk has released that buffer: at once for the delta-like
      // variants, whose preparation is the longer group; after the inverse for the diagonal variant, so that its
      // inverse runs while the chain works on innovations and read-out, not beside the next chunk's variances.
      const int irow = row & 63;
      auto emit_d1 = [&](auto store) {
        float Y[32];
        sm100::tmem_ld32(tmem + t_lane + Lay::T_D1 + 32 * half, Y);
        sm100::tmem_wait_ld();
        if (ell[s][kC - 1] >= -80.f) {
          const float Ai = Aex[s][irow];
          store(Y, [&](int jj) { return Ai * gcol[s][jj]; });
        } else {
          const float li = ell[s][irow];
          store(Y, [&](int jj) { return __expf(li - ell[s][jj]) * (delta_like(VAR) ? sB[s][jj] : 1.f); });
        }
      };
      auto emit_attn = [&] {
        emit_d1([&](const float (&Y)[32], auto gam) {
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            float xa[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int jj = 32 * half + 8 * q8 + e;
              xa[e] = (jj <= irow) ? Y[8 * q8 + e] * gam(jj) : 0.f;
            }
            store8_f16(TAThi, sm100::sw128_chunk(64 + irow, 4 * half + q8), xa);
          }
        });
      };
      // ---------------------------------------------------------------- N (lanes 0..63) | Attn (lanes 64..127)
      if (!kLateAttn && qw >= 2) emit_attn();
      if (qw < 2) {
        emit_d1([&](const float (&Y)[32], auto gam) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            float v4[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int jj = 32 * half + e + u;
              v4[u] = (jj < irow) ? Y[e + u] * gam(jj) : 0.f;
            }
            *reinterpret_cast<float4*>(Nf + irow * LD + 32 * half + e) = make_float4(v4[0], v4[1], v4[2], v4[3]);
          }
        });
      }
      named_sync(kBarPrep, kGroup);

      // ---------------------------------------------------------------- T = (I + N)^-1 (fp32 scratch)
      chunk::invert_unit_lower_64(Nf, Tf, pt, [] { named_sync(kBarPrep, kGroup); });

      // ---------------------------------------------------------------- [T; Attn] and -T diag(A)
      if (kLateAttn) {
        if (c >= 1 && !prep_wait(&tat_free, (c - 1) & 1)) { aborted = true; break; }
        if (qw >= 2) emit_attn();
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int e = pt + 256 * hh;
        const int i = e >> 3, c8 = e & 7;
        const float4 lo4 = *reinterpret_cast<const float4*>(Tf + i * LD + 8 * c8);
        const float4 hi4 = *reinterpret_cast<const float4*>(Tf + i * LD + 8 * c8 + 4);
        const float tv[8] = {lo4.x, lo4.y, lo4.z, lo4.w, hi4.x, hi4.y, hi4.z, hi4.w};
        float xt[8], xd[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int jj = 8 * c8 + u;
          xt[u] = (jj < i) ? tv[u] : (jj == i ? 1.f : 0.f);
          xd[u] = -xt[u] * Aex[s][jj];
        }
        store8_f16(TAThi, sm100::sw128_chunk(i, c8), xt);
        store8_f16(TADs, sm100::sw128_chunk(i, c8), xd);
      }
      sm100::fence_async_smem();
      sm100::tc_fence_before();
      named_sync(kBarPrep, kGroup);
      sm100::tc_fence_after();

      if (leader) sm100::mbar_arrive(&prep_done[s]);
    }
    if (VAR == kIso && !aborted && gw == 4 && lane == 0) P.p[bh] = c_iso;
  }

  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 0) sm100::tmem_dealloc(tmem, Lay::TMEM_COLS);
}

template <int VAR, int DT>
cudaError_t launch_ws_typed(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const Params& p, int BH,
                            cudaStream_t stream) {
  using Lay = WsLayout<VAR>;
  cudaError_t e =
      cudaFuncSetAttribute(chunk_scan_ws_kernel<VAR, DT>, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::SMEM);
  if (e != cudaSuccess) return e;
  chunk_scan_ws_kernel<VAR, DT><<<BH, kThreads, Lay::SMEM, stream>>>(q, k, v, p);
  return cudaGetLastError();
}

template <int DT>
cudaError_t launch_ws_dim(kdn_variant variant, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          const Params& p, int BH, cudaStream_t stream) {
  if (variant == KDN_KALMAN_FULL) return launch_ws_typed<kFull, DT>(tq, tk, tv, p, BH, stream);
  if (variant == KDN_KALMAN_ISO) return launch_ws_typed<kIso, DT>(tq, tk, tv, p, BH, stream);
  if (variant == KDN_KALMAN_DIAG) return launch_ws_typed<kDiag, DT>(tq, tk, tv, p, BH, stream);
  return launch_ws_typed<kDelta, DT>(tq, tk, tv, p, BH, stream);
}

}  // namespace

cudaError_t launch_chunk_ws(kdn_variant variant, const kdn_dims& d, const ChunkArgs& a, const float* gains,
                            cudaStream_t stream) {
  if (d.dk != d.dv || (d.dk != 64 && d.dk != D)) return cudaErrorInvalidValue;
  if (variant == KDN_KALMAN_FULL && gains == nullptr) return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv;
  if (!make_bf16_tmap(&tq, a.q, a.BH, a.L, d.dk) || !make_bf16_tmap(&tk, a.k, a.BH, a.L, d.dk) ||
      !make_bf16_tmap(&tv, a.v, a.BH, a.L, d.dv))
    return cudaErrorInvalidValue;
  Params p{};
  p.beta = a.beta, p.a = a.a, p.r = a.r, p.qn = a.qn, p.qn_scalar = a.qn_scalar, p.gains = gains;
  p.S = a.S, p.o = a.o, p.m = a.m, p.out_dtype = a.out_dtype, p.L = a.L, p.status = a.status;
  p.s_cols = a.state_cols == 0 ? d.dv : a.state_cols;
  if (p.s_cols != d.dv && !(d.dk == 64 && p.s_cols == 2 * d.dv)) return cudaErrorInvalidValue;
  // diagonal: the variances, [BH, d]; isotropic: the uncertainty scalar c, [BH]
  if (variant == KDN_KALMAN_DIAG || variant == KDN_KALMAN_ISO) p.p = a.P;
  return d.dk == D ? launch_ws_dim<D>(variant, tq, tk, tv, p, a.BH, stream)
                   : launch_ws_dim<64>(variant, tq, tk, tv, p, a.BH, stream);
}

}  // namespace kdn
