// Internal launch interface between the C-ABI layer (kdn_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace kdn {

// Per-token S-side scan: o, m and the final S for gains g_t given either as
// beta_t k_t (delta rule) or read from a precomputed fp32 gain array.
struct SeqScanArgs {
  const void* q;
  const void* k;
  const void* v;
  int in_dtype;
  int out_dtype;
  const float* beta;   // delta: [BH, L]
  const float* a;      // [BH, L] or nullptr
  const float* gains;  // Kalman: [BH, L, dk] fp32, or nullptr for the delta rule
  float* S;            // [BH, dk, dv]
  void* o;             // [BH, L, dv], or nullptr (not written)
  float* m;            // [BH, L] or nullptr
  int BH;
  int L;
  // backward pass support (both optional): the state at the start of every ckpt_every-token chunk,
  // [BH, ceil(L / ckpt_every), dk, dv], and the residual norms ||e_t||, [BH, L]
  float* S_ckpt = nullptr;
  float* enorm = nullptr;
  int ckpt_every = 64;  // a multiple of 16
};

// Backward pass of the gated delta rule scan (chunks of 32 tokens).
struct DeltaBwdArgs {
  const void* q;
  const void* k;
  const void* v;
  int in_dtype;
  const float* beta;    // [BH, L]
  const float* a;       // [BH, L] or nullptr (a_t = 1)
  const float* dO;      // [BH, L, dv] fp32 upstream gradient of o
  const float* dm;      // [BH, L] or nullptr
  const float* dS_L;    // [BH, dk, dv] or nullptr
  const float* S_ckpt;  // [BH, ceil(L / 32), dk, dv]: the state entering every 32-token chunk
  const float* enorm;   // [BH, L]: ||e_t|| of the forward
  float* dq;            // [BH, L, dk], zeroed: accumulated over value-column blocks
  float* dk;            // [BH, L, dk], zeroed
  float* dv;            // [BH, L, dv]
  float* dbeta;         // [BH, L], zeroed
  float* da;            // [BH, L], zeroed, or nullptr
  float* dS0;           // [BH, dk, dv]
  int BH;
  int L;
  // given gains instead of beta_t k_t (diagonal Kalman): gains [BH, L, dk] in, dgain [BH, L, dk] (zeroed) out;
  // beta and dbeta are then unused
  const float* gains = nullptr;
  float* dgain = nullptr;
};
constexpr int kDeltaBwdChunk = 32;
cudaError_t launch_delta_bwd(int dk, int dv, const DeltaBwdArgs& args, cudaStream_t stream);

// Uncertainty side of the isotropic-Kalman backward (one warp per head).
struct IsoBwdArgs {
  const void* k;        // [BH, L, dk]
  int in_dtype;
  const float* a;       // [BH, L] or nullptr
  const float* r;       // [BH, L]
  const float* qn;      // [BH, L] or nullptr (qn_scalar)
  float qn_scalar;
  const float* c0;      // [BH] or nullptr (1)
  float* beta;          // [BH, L] forward: beta_t
  float* cprev;         // [BH, L] forward: c before token t
  float* knorm2;        // [BH, L] forward: ||k_t||^2
  const float* dbeta;   // [BH, L] backward: dLoss/dbeta_t from the memory backward
  const float* dc_L;    // [BH] or nullptr: upstream gradient of the final c
  float* dk;            // [BH, L, dk] in/out: the key terms are added
  float* da;            // [BH, L] in/out or nullptr: the gate terms are added
  float* dr;            // [BH, L] out
  float* dqn;           // [BH, L] out
  float* dc0;           // [BH] out
  int L;
  int dk_dim;           // d_k
};
cudaError_t launch_iso_forward(const IsoBwdArgs& args, int BH, cudaStream_t stream);
cudaError_t launch_iso_backward(const IsoBwdArgs& args, int BH, cudaStream_t stream);

// Uncertainty side of the diagonal-Kalman backward (one warp per head, lanes over the coordinates).
struct DiagBwdArgs {
  const void* k;        // [BH, L, dk]
  int in_dtype;
  const float* a;       // [BH, L] or nullptr
  const float* r;       // [BH, L]
  const float* qn;      // [BH, L] or nullptr (qn_scalar)
  float qn_scalar;
  const float* p0;      // [BH, dk] or nullptr (1)
  float* gains;         // [BH, L, dk] forward: g_t = p^- o k / s
  float* pprev;         // [BH, L, dk] forward: p before token t
  const float* dgain;   // [BH, L, dk] backward: dLoss/dg_t from the memory backward
  const float* dp_L;    // [BH, dk] or nullptr: upstream gradient of the final p
  float* dk;            // [BH, L, dk] in/out: the key terms are added
  float* da;            // [BH, L] in/out or nullptr: the gate terms are added
  float* dr;            // [BH, L] out
  float* dqn;           // [BH, L] out
  float* dp0;           // [BH, dk] out
  int L;
  int dk_dim;           // d_k
};
cudaError_t launch_diag_forward(const DiagBwdArgs& args, int BH, cudaStream_t stream);
cudaError_t launch_diag_backward(const DiagBwdArgs& args, int BH, cudaStream_t stream);

// Covariance side of the full-Kalman backward: the forward keeps the per-token gains and P at every 32-token
// block start; the backward recomputes each block and walks it in reverse with M = Pb + Pb^T.
struct FullBwdArgs {
  const void* k;        // [BH, L, d]
  int in_dtype;
  const float* a;       // [BH, L] or nullptr
  const float* r;       // [BH, L]
  const float* qn;      // [BH, L] or nullptr (qn_scalar)
  float qn_scalar;
  const float* P0;      // [BH, d, d] or nullptr (I)
  float* gains;         // [BH, L, d] forward: g_t = u_t / s_t
  float* ckpt;          // scratch [BH, nblk, d, d]: P at every block start (thread order)
  float* scr_P;         // scratch [BH, 32, d, d]: P before every token of the block being walked
  const float* dgain;   // [BH, L, d] backward: dLoss/dg_t from the memory backward
  const float* dP_L;    // [BH, d, d] or nullptr: upstream gradient of the final P
  float* dk;            // [BH, L, d] in/out: the key terms are added
  float* da;            // [BH, L] in/out or nullptr: the gate terms are added
  float* dr;            // [BH, L] out
  float* dqn;           // [BH, L] out
  float* dP0;           // [BH, d, d] out: the gradient for a symmetric P0
  unsigned* status;     // the call's status word (a non-positive or non-finite s)
  int L;
  int d;                // d_k: 16, 32, 64 or 128
};
size_t full_backward_scratch_bytes(int BH, int L, int d);
void full_backward_bind_scratch(FullBwdArgs& args, void* scratch, int BH);
cudaError_t launch_full_cov_forward(const FullBwdArgs& args, int BH, cudaStream_t stream);
cudaError_t launch_full_cov_backward(const FullBwdArgs& args, int BH, cudaStream_t stream);

// Sequence-parallel covariance side of the full-Kalman scan (chunks of 64 tokens): the covariance entering
// every run of cps chunks, through the chunks' Riccati transfer matrices.
struct RiccatiArgs {
  const void* k;        // [BH, L, d] bf16
  const float* a;       // [BH, L] or nullptr
  const float* r;       // [BH, L]
  const float* qn;      // [BH, L] or nullptr (qn_scalar)
  float qn_scalar;
  const float* P0;      // [BH, d, d]
  float* map_g;         // [BH, nch, 64, 64] scratch: G^T of every chunk
  float* map_u;         // [BH, nch, 64] scratch
  float* map_ab;        // [BH, nch, 64, 2] scratch: alpha_t, beta_t
  float* xy;            // [BH, runs, 2d, d] scratch: [X; Y] entering every run
  float* P_starts;      // [BH, runs, d, d] out: the covariance entering every run
  unsigned* status;
  int BH;
  int L;
  int cps;              // chunks per run; runs = ceil(nch / cps)
};
// Bytes of the scratch above (map_g, map_u, map_ab, xy, P_starts, each 256-byte aligned).
size_t riccati_scratch_bytes(int d, int BH, int L, int cps);
cudaError_t launch_riccati_starts(int d, const RiccatiArgs& args, cudaStream_t stream);

// Per-token Kalman gain recursions (covariance side; independent of v and S).
struct GainArgs {
  const void* k;
  int in_dtype;
  const float* a;   // [BH, L] or nullptr
  const float* r;   // [BH, L]
  const float* qn;  // [BH, L] or nullptr
  float qn_scalar;
  float* P;         // full: [BH, dk, dk]
  float* p;         // diagonal: [BH, dk]
  float* gains;     // out: [BH, L, dk]
  unsigned* status;
  int BH;
  int L;
};

struct DecodeArgs {
  const void* q;
  const void* k;
  const void* v;
  int in_dtype;
  int out_dtype;
  const float* beta;  // delta: [BH]
  const float* a;     // [BH] or nullptr
  const float* r;     // diagonal: [BH]
  float qn_scalar;
  float* S;           // [BH, dk, dv]
  float* p;           // diagonal: [BH, dk]; isotropic: c, [BH]
  void* o;            // [BH, dv]
  float* m;           // [BH] or nullptr
  int BH;
};

// Isotropic-Kalman prologue: per-token write strengths beta_t from one uncertainty scalar per head.
struct IsoArgs {
  const void* k;     // [BH, L, dk]
  int in_dtype;
  const float* a;    // [BH, L] or nullptr
  const float* r;    // [BH, L]
  const float* qn;   // [BH, L] or nullptr
  float qn_scalar;
  float* c;          // [BH] in/out
  float* beta;       // out: [BH, L]
  unsigned* status;
  int L;
};

// Surprise-cache read: top-w exact cache by m, sharpened softmax over cache, causal block and a sink.
struct HolaArgs {
  const void* q;          // [BH, L, dk]
  const void* k;          // [BH, L, dk]
  const void* v;          // [BH, L, dv]
  int in_dtype;
  const float* m;         // [BH, L] surprise
  const float* gamma_q;   // [dk]
  const float* gamma_k;   // [dk]
  const float* sink;      // [H]
  float* o;               // [BH, L, dv] fp32
  int* cache;             // [BH, w] final cache token indices, or nullptr
  int H;
  int L;
  int block;              // 16, 32 or 64
  int w;                  // 1..64
  unsigned* status;       // device status word (bounded-wait timeouts)
  // [BH, ceil(L / 64), 64] scratch, or nullptr: the cache token indices each block reads (tensor-core path:
  // every block's cache is chosen first, then all blocks are read in parallel)
  int* cidx = nullptr;
};

// Segment-parallel scan (P segments per head): uncertainty maps and starts, start states, chaining.
struct SegArgs {
  int P;                  // segments per head (L % P == 0)
  int L;                  // tokens per head
  // diagonal-Kalman uncertainty at the segment starts
  const void* k;          // [BH, L, dk]
  int in_dtype;
  const float* a;         // [BH, L] or nullptr
  const float* r;         // [BH, L]
  const float* qn;        // [BH, L] or nullptr
  float qn_scalar;
  const float* p0;        // [BH, dk] p before the first token
  float4* maps;           // [BH P, dk] composed map of each segment (slot P - 1 unused)
  float* pcopy[3];        // [BH P, dk] each: p at every segment start
  int ncopy;
  // memory state
  const float* S;         // [BH, d, d] the caller's start state
  float* Sz;              // [BH P, d, d] segment end states from S0 = 0 (aug: [BH P, d, 2 d], [B | M])
  float* SI;              // [BH P, d, d] segment end states from S0 = I (aug: unused)
  int aug;                // 1: one run on [S | M] from [0 | I] gave B and M side by side
  float* Sc;              // [BH P, d, d] out: the true start state of every segment
  unsigned* status;
};

cudaError_t launch_seg_uncertainty(int dk, const SegArgs& args, int BH, cudaStream_t stream);
cudaError_t launch_seg_init(int d, const SegArgs& args, int BH, cudaStream_t stream);
cudaError_t launch_seg_combine(int d, const SegArgs& args, int BH, cudaStream_t stream);

cudaError_t launch_seq_scan(int dk, int dv, const SeqScanArgs& args, cudaStream_t stream);
cudaError_t launch_hola_read(int dk, int dv, const HolaArgs& args, int BH, cudaStream_t stream);
// tensor-core variant (bf16, d_k = d_v = 128, blocks of 64); launch_hola_read picks it when it applies
bool hola_tc_supported(int dk, int dv, int in_dtype, int block);
cudaError_t launch_hola_read_tc(const HolaArgs& args, int BH, cudaStream_t stream);
cudaError_t launch_iso_beta(int dk, const IsoArgs& args, int BH, cudaStream_t stream);
cudaError_t launch_kalman_full_gains(int dk, const GainArgs& args, cudaStream_t stream);
cudaError_t launch_kalman_diag_gains(int dk, const GainArgs& args, cudaStream_t stream);
// mode: 0 delta, 1 diagonal Kalman (p = [BH, dk]), 2 isotropic Kalman (p = c, [BH])
cudaError_t launch_decode(int dk, int dv, int mode, const DecodeArgs& args, cudaStream_t stream);

}  // namespace kdn
