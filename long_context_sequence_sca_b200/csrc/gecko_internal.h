// Internal interface between the C-ABI host code and the kernel launchers.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace gecko {

constexpr int kF32 = 0;
constexpr int kBF16 = 1;

// One validated forward call.
struct Problem {
  const void *q, *k, *v, *qm, *km;
  void *out_sca, *out_mem;
  int64_t B, H, T, c, d;
  int S;
  int dtype;
  int* status;        // device status word
  // Continuation of a longer sequence (all zero for a fresh start):
  int64_t koff = 0;              // rows of the previous chunk prepended to k and v per head (0 or c)
  const float* state0 = nullptr; // [BH, 2 d^2 + d] carried state (device): M'_prev, M'_cur, log z
  float* lse = nullptr;          // [BH, T] SCA row log-sum-exp (natural log), written if set
  void* out_sca_lo = nullptr;    // [BH, T, d] rounding residual of out_sca (O - rounded O), written if set
};

// Floats per (b, h) in a carried state record: M'_prev, M'_cur (d x d each), log z (d).
inline int64_t state_floats(int64_t d) { return 2 * d * d + d; }

// Device workspace carved out of one allocation (fp32 but for Mimg).
struct Workspace {
  float2* part;  // [BH, T / R, d]  (max, sum exp(x - max)) of K_m per block of R rows
  float* lse;    // [BH, S, d]  log of per-chunk exp-sums of K_m
  float* logz;   // [BH, S, d]  log z^s
  float* ratio;  // [BH, S, d]  z^{s-1} / z^s  (0 for s = 1)
  float* rho;    // [BH, S, d]  e_s / z^s = exp(lse_s - log z^s)
  float* Bm;     // [BH, S, d, d]  Phi~_s^T V_s    (Phi~_s = exp(Km_s - lse_s))
  float* Cm;     // [BH, S, d, d]  Phi~_s^T Psi_s
  float* Mst;    // [BH, S+1, d, d]  M'_1 .. M'_{S+1}
  // [BH, S+1, d * d] bf16 bits: image s is the readout's B operand for
  // chunk s (0-based), i.e. M'_{s-1} (1-based) = Mst[s - 1] for s >= 1 and
  // the carried M'_prev for s = 0, as bf16 in the 128-byte-swizzled
  // MN-major layout (64-column boxes of d rows).  Written by the carry.
  uint16_t* Mimg;
  // [BH, S, d * d] bf16 bits: Cm_s rounded to bf16 in the K-major
  // 128-byte-swizzled operand layout (rows f, K = g), written by the forward
  // chunk kernel at d = 128 and read by the tensor-core carry.
  uint16_t* Cimg;
  // [BH, S]: 1 where the fused statistics' first-tile reference was
  // outgrown and the chunk has to be redone (written for every chunk).
  int* flags;
};

// Column slices of the sequential carries: as wide as still gives about one
// CTA per SM (every CTA runs all S steps, so a second wave would double the
// time).
inline int carry_slice(int64_t BH, int D) {
  for (int jc : {32, 16})
    if (BH * (D / jc) >= 100) return jc;
  return 8;
}

// Rows per block of the partial K_m statistics (divides c).
inline int stats_block_rows(int64_t c) { return c % 128 == 0 ? 128 : 64; }

// Bytes needed by a Workspace, each region 256-byte aligned.
size_t workspace_bytes(int64_t BH, int64_t T, int64_t c, int64_t d);
Workspace carve_workspace(void* base, int64_t BH, int64_t T, int64_t c, int64_t d);

// CUDA-core kernels (any dtype, any c % 64 == 0).
cudaError_t launch_awm_stats(const Problem& p, const Workspace& w, cudaStream_t st);   // lse + log z prefix
cudaError_t launch_awm_prefix(const Problem& p, const Workspace& w, cudaStream_t st);  // log z prefix from lse
cudaError_t launch_awm_chunk_simt(const Problem& p, const Workspace& w, cudaStream_t st);
// images: also write the readout operand images (Workspace::Mimg)
cudaError_t launch_awm_carry(const Problem& p, const Workspace& w, cudaStream_t st, bool images = false);
cudaError_t launch_awm_readout_simt(const Problem& p, const Workspace& w, cudaStream_t st);
cudaError_t launch_sca_simt(const Problem& p, cudaStream_t st);

// Streaming multiprocessors of the current device (queried once).
int sm_count();

// Tensor-core (tcgen05 + TMEM + TMA) kernels, bf16 with c % 128 == 0.
bool tc_supported(const Problem& p);
cudaError_t launch_sca_tc(const Problem& p, cudaStream_t st);
// parts > 1: that many CTAs share each chunk and add into Bm, Cm (zeroed
// here), and the bf16 image of Cm is made by a separate pass
cudaError_t launch_awm_chunk_tc(const Problem& p, const Workspace& w, cudaStream_t st, int parts = 1);
// the chunk products with each chunk's log-sum-exp (Workspace::lse) computed
// in the same pass (two launches: against the first tile's reference, then a
// redo of the chunks flagged in Workspace::flags)
cudaError_t launch_awm_chunk_tc_stats(const Problem& p, const Workspace& w, cudaStream_t st);
cudaError_t launch_awm_readout_tc(const Problem& p, const Workspace& w, cudaStream_t st);
// The carry on the tensor cores (d = 128; bf16 hi + lo operands, ~fp32 products)
cudaError_t launch_awm_carry_tc(const Problem& p, const Workspace& w, cudaStream_t st, bool images);
// Bm, Cm with each computed operand as bf16 hi + lo (near-fp32 products for the backward)
cudaError_t launch_awm_chunk_tc_split(const Problem& p, const Workspace& w, cudaStream_t st);
// E_s = psi(Qm_s)^T dO_m,s for chunks 3..S, hi + lo operands
cudaError_t launch_awm_bwd_e_tc(const Problem& p, const void* dout_mem, float* E, cudaStream_t st);

// ------------------------------------------------------------ backward --

// One validated backward call: the forward's inputs (f.q .. f.km, sizes,
// dtype), the forward's SCA output and row log-sum-exp, the output
// gradients, and the input gradients to write (all [B, H, T, d] dtype).
struct BwdProblem {
  Problem f;
  const void* out_sca;
  const void* out_sca_lo;   // may be null
  const float* lse;
  const void *dout_sca, *dout_mem;
  void *dq, *dk, *dv, *dqm, *dkm;
};

struct BwdWorkspace {
  float* delta;   // [BH, T]  rowsum(dO * O) of SCA
  float* nlse2;   // [BH, T]  -log2(e) * (SCA row log-sum-exp)
  float* E;       // [BH, S, d, d]  psi(Qm_s)^T dO_m,s
  float* G;       // [BH, S+1, d, d]  G_s = dLoss/dM'_s, s = 1..S+1
  float* dl;      // [BH, S, d]  dLoss/d log e_s
  float* dv_awm;  // [BH, T, d]  AWM part of dV
  float* W;       // [BH, S, d, d]  W_s = M'_s G_{s+1}^T
};

size_t bwd_workspace_bytes(int64_t BH, int64_t T, int64_t c, int64_t d);
BwdWorkspace carve_bwd_workspace(void* base, int64_t BH, int64_t T, int64_t c, int64_t d);
cudaError_t launch_sca_bwd_delta(const BwdProblem& b, const BwdWorkspace& w, cudaStream_t st);
// part 0: dK and dV (adding the AWM part of dV); part 1: dQ
cudaError_t launch_sca_bwd_simt(const BwdProblem& b, const BwdWorkspace& w, cudaStream_t st, int part);
cudaError_t launch_sca_bwd_tc(const BwdProblem& b, const BwdWorkspace& w, cudaStream_t st, int part);  // bf16, tc_supported
// tc: the per-chunk K_m / V gradients on the tensor cores (bf16, tc_supported)
cudaError_t launch_awm_bwd(const BwdProblem& b, const Workspace& fw, const BwdWorkspace& w, cudaStream_t st,
                           bool tc);
cudaError_t launch_awm_bwd_chunk_tc(const BwdProblem& b, const Workspace& fw, const BwdWorkspace& w,
                                    cudaStream_t st);
cudaError_t launch_awm_bwd_readout_tc(const BwdProblem& b, const Workspace& fw, cudaStream_t st);

// -------------------------------------------------- context parallelism --

cudaError_t launch_set_identity(float* dst, int64_t stride, int d, int64_t BH, cudaStream_t st);
// out[bh * sd + f] = logsumexp_{j < rank} lsum[j, bh, f]  (-inf for rank 0)
cudaError_t launch_cp_logz(const float* lsum, float* out, int rank, int64_t BH, int d, int64_t sd, cudaStream_t st);
// out[bh * sd] = M'_prev, out[bh * sd + d*d] = M'_in from the maps of ranks < rank
cudaError_t launch_cp_compose(const float* maps, float* out, int rank, int64_t BH, int d, int64_t sd,
                              cudaStream_t st);

// ---------------------------------------------------------------- CEMA --

// One validated CEMA call: x, y [B, L, D] (dtype); alpha, delta, theta,
// beta [D, 16] fp32; eta [D, 16, 2] fp32; reset [B, L] uint8 or null;
// state_in / state_out [B, D, 16, 2] fp32 or null (device).
struct CemaProblem {
  const void* x;
  void* y;
  const float *alpha, *delta, *theta, *beta, *eta;
  const uint8_t* reset;
  const float* state_in;
  float* state_out;
  int64_t B, L, D;
  int dtype;
  int* status;   // device status word (bounded waits that ran out)
};

struct CemaWorkspace {
  float2* Bc;            // [B, C, D, 16]  end state of each chunk scanned from zero
  float2* Hin;           // [B, C, D, 16]  state entering each chunk
  uint8_t* chunk_reset;  // [B, C]  1 if the chunk holds a document start
};

int cema_hidden();                       // hidden dimensions per feature (16)
int64_t cema_chunks(int64_t L);          // chunks of the scan
size_t cema_workspace_bytes(int64_t B, int64_t L, int64_t D);
CemaWorkspace carve_cema_workspace(void* base, int64_t B, int64_t L, int64_t D);
cudaError_t launch_cema(const CemaProblem& p, const CemaWorkspace& w, cudaStream_t st);

// ------------------------------------------------ timestep decay norm --

// One validated call: x, y [B, L, D] (dtype); gamma, bias [D] fp32 (device);
// G groups of D / G features.
struct NormProblem {
  const void* x;
  void* y;
  const float *gamma, *bias;
  int64_t B, L, D, G;
  float beta1, beta2, eps;
  int dtype;
};

struct NormWorkspace {
  float2* stats;    // [B, L, G]  (mean, variance) of each group
  float2* affine;   // [B, L, G]  (scale, shift) from the decayed statistics
};

size_t tdnorm_workspace_bytes(int64_t B, int64_t L, int64_t G);
NormWorkspace carve_tdnorm_workspace(void* base, int64_t B, int64_t L, int64_t G);
cudaError_t launch_tdnorm(const NormProblem& p, const NormWorkspace& w, cudaStream_t st);

}  // namespace gecko
