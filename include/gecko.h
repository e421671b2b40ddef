/*
 * gecko.h - C ABI of the Gecko fused forward for NVIDIA B200 (sm_100a).
 *
 * The library computes, per (batch b, head h), the two attention parts of a
 * Gecko layer ("Gecko: An Efficient Neural Architecture Inherently Processing
 * Sequences with Arbitrary Lengths", arXiv 2601.06463):
 *
 *   Sliding Chunk Attention (SCA)  - Gecko digest (paper.rainbus.top),
 *     method step details, step 3; paperlayer.ai summary, section 3.2:
 *       O_s = softmax(Q_s [K_{s-1}; K_s]^T) [V_{s-1}; V_s]
 *     for chunk s of c tokens.  Scale 1 (no 1/sqrt(d)), causal inside the
 *     current chunk, all c keys of the previous chunk visible, and chunk 1
 *     attends only to itself.
 *
 *   Adaptive Working Memory (AWM)  - digest, core method (online-softmax
 *     kernel) and step details, steps 4-5; paperlayer.ai summary, section
 *     3.3 and Appendix A:
 *       z^s   = sum_{t<=s} sum_{i<=c} exp(Km_{t,i})            (per feature)
 *       phi^s(Km_s) = exp(Km_s) / z^s,   psi(x) = softmax over features
 *       M'_1 = 0,
 *       M'_s = (z^{s-2}/z^{s-1}) (.) M'_{s-1}
 *              + phi^{s-1}(Km_{s-1})^T (V_{s-1} - psi(Km_{s-1}) M'_{s-1})
 *       O_m,s = psi(Qm_s) M'_{s-1}        (M'_0 := 0: chunks 1, 2 read 0)
 *     The z-ratio scales row f (key feature f) of M'.
 *
 *   The layer output is out_sca + out_mem (digest, step 5); the two parts
 *   are returned separately and the caller adds them.
 *
 * Layout: every tensor is caller-owned, contiguous, row-major [B, H, T, d]
 * (d innermost) in device memory, all of one dtype, each base address
 * 16-byte aligned.  The value dimension equals d.
 *
 * Execution is asynchronous on `stream` (a cudaStream_t; NULL means the
 * legacy default stream).  Argument errors are detected on the host before
 * anything is launched or written.  Faults inside a kernel surface at the
 * caller's next synchronisation.  Every device-side wait is bounded in time;
 * a wait that runs out sets a device status word read by
 * gecko_device_status().
 *
 * Environment (read at each call; for tests and cross-checks):
 *   GECKO_KERNELS=simt    run the CUDA-core kernels for every dtype instead of
 *                         the tensor-core ones (a second GPU implementation).
 *   GECKO_CHUNK_PARTS=k   use k CTAs per chunk for the AWM chunk products
 *                         (1 <= k <= c / 64, tensor-core path only) instead
 *                         of the library's choice;
 *                         with one CTA per chunk the chunk kernel also computes
 *                         the chunk's K_m statistics.
 *   GECKO_FAIL_ALLOC=1    make every workspace allocation fail
 *                         (GECKO_ERR_ALLOC), to test callers' error paths.
 *   GECKO_CEMA_PLAIN=1    load the CEMA inputs with plain loads instead of TMA.
 * Other values of these variables are ignored.
 */
#ifndef GECKO_H
#define GECKO_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* dtype codes */
#define GECKO_F32  0   /* fp32 in, fp32 out, fp32 arithmetic (SIMT FMA) */
#define GECKO_BF16 1   /* bf16 in, bf16 out, fp32 accumulation            */

/* status codes */
#define GECKO_OK            0
#define GECKO_ERR_ARG       1  /* null pointer, bad dtype, size < 1, mismatched state query */
#define GECKO_ERR_SHAPE     2  /* T % c != 0, c % 64 != 0, d not in {64, 128}, size overflow */
#define GECKO_ERR_ALIGN     3  /* a tensor base address is not 16-byte aligned              */
#define GECKO_ERR_ALLOC     4  /* the library workspace could not be allocated              */
#define GECKO_ERR_CUDA      5  /* a CUDA runtime call or kernel launch failed               */
#define GECKO_ERR_NO_STATE  6  /* gecko_awm_state before any forward on this device         */
#define GECKO_ERR_TIMEOUT   7  /* a bounded device-side wait ran out                        */
#define GECKO_ERR_LIMIT     8  /* workspace above the fixed scratch of the no-allocation entry */

/*
 * gecko_sca_awm_forward - fused SCA + AWM forward of one layer.
 *
 *   q, k, v, qm, km : [B, H, T, d] inputs (device), dtype `dtype`.
 *                     q, k feed SCA; qm, km feed AWM; v feeds both.
 *   out_sca, out_mem: [B, H, T, d] outputs (device), dtype `dtype`;
 *                     fully overwritten.  They must not alias an input.
 *   B, H, T, c, d   : batch, heads, tokens, chunk size, head dim.
 *                     Requires B, H, T >= 1, c >= 64, c % 64 == 0,
 *                     T % c == 0, d in {64, 128}, B * H <= 65535,
 *                     T / c <= 65535 and T < 2^31 - 256 (else
 *                     GECKO_ERR_SHAPE).
 *   dtype           : GECKO_F32 or GECKO_BF16.
 *   stream          : cudaStream_t used for every launch and copy.
 *
 * Ownership: the library keeps one workspace per device (log z per chunk,
 * per-chunk memory matrices, the carried state).  It grows on demand with
 * stream-ordered allocation on `stream` and lives until gecko_release().
 * Forwards of any kind (this one, _continue, _train, _noalloc, the
 * context-parallel segment calls, and the backward's rebuild) must not
 * overlap on the GPU on one device: besides the workspace they share the
 * SCA kernel's work-unit counter and the device status word, so overlapping
 * calls lose or repeat work.  Every call starts from M'_1 = 0 (no initial
 * state).
 *
 * Returns GECKO_OK or an error code; the message is in gecko_last_error().
 */
int gecko_sca_awm_forward(const void* q, const void* k, const void* v,
                          const void* qm, const void* km,
                          void* out_sca, void* out_mem,
                          int64_t B, int64_t H, int64_t T, int64_t c, int64_t d,
                          int dtype, void* stream);

/*
 * gecko_sca_awm_forward_train - gecko_sca_awm_forward that also keeps what
 * the backward needs from SCA: the natural-log sum of exp of each query
 * row's visible scores (the softmax normaliser of SCA, Gecko digest, method
 * step details, step 3).
 *
 *   lse        : [B, H, T] fp32 (device), 16-byte aligned; fully overwritten.
 *   out_sca_lo : NULL, or [B, H, T, d] dtype (device), 16-byte aligned: the
 *                rounding residual of out_sca (the exact output minus the
 *                stored one, rounded to dtype; zero for GECKO_F32).  The
 *                backward's row term rowsum(dO * O) cancels strongly at long
 *                windows, and with bf16 O alone its error dominates dq.
 *
 * Everything else as gecko_sca_awm_forward (same outputs, bit for bit).
 */
int gecko_sca_awm_forward_train(const void* q, const void* k, const void* v,
                                const void* qm, const void* km,
                                void* out_sca, void* out_mem, float* lse, void* out_sca_lo,
                                int64_t B, int64_t H, int64_t T, int64_t c, int64_t d,
                                int dtype, void* stream);

/*
 * gecko_sca_awm_backward - gradients of one fresh-sequence forward with
 * respect to q, k, v, qm, km, given the gradients of its two outputs.  The
 * pages print no backward; this is the chain rule of the forward above (SCA:
 * digest step 3; AWM: digest core method and steps 4-5, paperlayer.ai
 * summary section 3.3 and Appendix A).  As the summary's appendix B.1
 * (backward pass) describes, only chunk-boundary states are needed: they
 * are rebuilt here from qm, km, v, so the forward keeps nothing but lse.
 *
 *   q, k, v, qm, km : the forward's inputs, [B, H, T, d] dtype (device).
 *   out_sca, out_sca_lo, lse : the forward's SCA output, its residual
 *                     (may be NULL: then O is taken as out_sca alone) and
 *                     lse (gecko_sca_awm_forward_train).
 *   dout_sca, dout_mem : gradients of out_sca and out_mem, [B, H, T, d].
 *   dq, dk, dv, dqm, dkm : [B, H, T, d] dtype (device), fully overwritten;
 *                     dv sums the SCA and AWM parts (v feeds both).  They
 *                     must not alias each other or any input.
 *   All pointers 16-byte aligned; same size constraints as the forward.
 *   The gradient of the exported state (M'_{S+1}, log z^S) is taken as zero.
 *
 * Ownership: a second per-device workspace (row statistics, per-chunk
 * state gradients, the AWM part of dV in fp32) grows like the forward's
 * and lives until gecko_release().  The call recomputes the forward's AWM
 * workspace, so gecko_awm_state afterwards reports this sequence's state.
 * Errors as gecko_sca_awm_forward.
 */
int gecko_sca_awm_backward(const void* q, const void* k, const void* v,
                           const void* qm, const void* km,
                           const void* out_sca, const void* out_sca_lo, const float* lse,
                           const void* dout_sca, const void* dout_mem,
                           void* dq, void* dk, void* dv, void* dqm, void* dkm,
                           int64_t B, int64_t H, int64_t T, int64_t c, int64_t d,
                           int dtype, void* stream);

/*
 * gecko_sca_awm_forward_continue - the same forward for one segment of a
 * longer sequence, so a sequence of any length runs in pieces whose outputs
 * equal those of one call over the whole sequence (up to rounding).  The AWM
 * state is what the pages carry from chunk to chunk (Gecko digest, core
 * method: z^s accumulates over all history; method step details, step 4:
 * M'_s is updated from M'_{s-1}; paperlayer.ai summary, section 3.3: memory
 * updates operate chunk by chunk), and SCA needs the previous chunk's keys
 * and values (step 3).
 *
 *   state_in == NULL: a fresh sequence.  k and v are [B, H, T, d]; identical
 *     to gecko_sca_awm_forward.
 *   state_in != NULL: a continuation.  k and v are [B, H, c + T, d]: per
 *     (b, h), the c rows of the previous segment's last chunk followed by
 *     this segment's T rows.  state_in is the state_out of the previous
 *     segment.  q, qm, km, out_sca, out_mem stay [B, H, T, d].
 *   state_out (may be NULL, may equal state_in): [B, H, 2 d^2 + d] fp32,
 *     per (b, h) M'_S (d x d), M'_{S+1} (d x d) and log z^S (d), in this
 *     segment's chunk numbering (S = T / c); device or host memory.
 *
 * Same constraints, ownership, workspace and errors as gecko_sca_awm_forward
 * (state_in is copied into the library's memory before use).  After the
 * call, gecko_awm_state reports this segment's state.
 */
int gecko_sca_awm_forward_continue(const void* q, const void* k, const void* v,
                                   const void* qm, const void* km,
                                   void* out_sca, void* out_mem,
                                   const float* state_in, float* state_out,
                                   int64_t B, int64_t H, int64_t T, int64_t c, int64_t d,
                                   int dtype, void* stream);

/*
 * gecko_sca_awm_forward_noalloc - the same forward as gecko_sca_awm_forward
 * (same arguments, kernels and results) for callers that must not allocate
 * device memory themselves or through this library: for example a plugin
 * whose host application's memory planner or pool owns all device memory,
 * or a latency-critical loop that cannot afford cudaMalloc's implicit
 * device-wide synchronisation.  The paper has no counterpart of this entry
 * point; it only changes where the working memory comes from.
 *
 * Working memory: instead of the growable workspace, every call uses one
 * fixed scratch array of GECKO_NOALLOC_SCRATCH_BYTES (80 MiB) that is part
 * of the library's device image; each GPU that loads the library holds it
 * until the process exits.  Inputs and outputs are still passed by the
 * caller.  The scratch needs
 *   4 * (2*BH*T/R*d + 4*BH*S*d + (3*S + 1)*BH*d*d + BH*S) + 2*(2*S + 1)*BH*d*d
 *   bytes (each of the eleven regions rounded up to 256 bytes; R = 128 if
 *   c % 128 == 0 else 64, S = T / c, BH = B * H),
 * e.g. B*H = 32, T = 32768, c = 4096, d = 128 needs about 79 MB.  Larger
 * problems are rejected with GECKO_ERR_LIMIT before anything is launched.
 * The call makes no cudaMalloc, cudaFree or other allocating call.
 *
 * The first call on a device resolves the scratch array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  All calls share the array and it keeps the
 * last call's contents (every region is fully written before it is read,
 * so nothing needs clearing).  A call must not overlap on the GPU with any
 * other forward on the same device, this entry point's or the allocating
 * ones: they share the array (no-allocation calls), the SCA kernel's
 * work-unit counter, which each SCA launch resets, and the device status
 * word, so overlapping calls lose or repeat work.
 * This entry point leaves the state reported by gecko_awm_state unchanged:
 * that state stays the one of the last allocating forward, continued
 * forward, training forward or backward on the device.
 */
#define GECKO_NOALLOC_SCRATCH_BYTES (80ull << 20)
int gecko_sca_awm_forward_noalloc(const void* q, const void* k, const void* v,
                                  const void* qm, const void* km,
                                  void* out_sca, void* out_mem,
                                  int64_t B, int64_t H, int64_t T, int64_t c, int64_t d,
                                  int dtype, void* stream);

/*
 * gecko_awm_state - copy the AWM state carried out of the most recent
 * gecko_sca_awm_forward or gecko_sca_awm_forward_continue call on the
 * current device: M_out [B, H, d, d] fp32 = M'_{S+1} (all S
 * chunks folded in, normalised by z^S; row = key feature) and logz_out
 * [B, H, d] fp32 = log z^S.  Pointers may be device or host memory
 * (cudaMemcpyDefault).  The copy is ordered on `stream`; the call returns
 * after the copy has completed.  Returns GECKO_ERR_NO_STATE if no forward
 * ran on this device, GECKO_ERR_ARG if B, H, d differ from that forward,
 * and GECKO_ERR_TIMEOUT if a kernel of that forward reported a timed-out
 * wait.  A gecko_sca_awm_backward call rebuilds the same state and counts as
 * such a forward; gecko_awm_segment_logsum and gecko_awm_segment_maps
 * invalidate it (GECKO_ERR_NO_STATE).
 */
int gecko_awm_state(float* M_out, float* logz_out,
                    int64_t B, int64_t H, int64_t d, void* stream);

/*
 * gecko_device_status - synchronise `stream`, then read and clear the
 * library's device status word on the current device.  Returns GECKO_OK,
 * GECKO_ERR_TIMEOUT if a kernel gave up on a bounded wait since the last
 * check, or GECKO_ERR_CUDA if the synchronisation failed.
 */
int gecko_device_status(void* stream);

/*
 * Measurement support.  gecko_timing_enable(1) makes every later forward
 * record CUDA events on its stream around its five stages:
 *   0 AWM statistics (per-chunk log exp-sums of K_m and the log z prefix),
 *   1 AWM chunk products (Phi^T V and Phi^T Psi per chunk),
 *   2 AWM carry (the sequential M' recurrence),
 *   3 AWM readout (psi(Q_m) M'_{s-1}),
 *   4 SCA.
 * gecko_timing_read() waits for the recorded forwards, writes the summed
 * milliseconds per stage into ms_per_stage[0 .. min(capacity, 5) - 1] and
 * the number of forwards into *n_calls, and clears the record.  Returns
 * GECKO_OK, GECKO_ERR_ARG for NULL buffers or capacity < 1, or
 * GECKO_ERR_CUDA.  Timing is off by default; when on it costs six event
 * records per forward.
 */
int gecko_timing_enable(int enable);
int gecko_timing_read(float* ms_per_stage, int capacity, int* n_calls);
/* The same for the backward (gecko_sca_awm_backward), five stages in order:
 * AWM state rebuild (stats, chunk products, carry), AWM reverse pass, SCA
 * row statistics, SCA dK/dV, SCA dQ. */
int gecko_timing_read_backward(float* ms_per_stage, int capacity, int* n_calls);

/*
 * gecko_cema_forward - CEMA, the complex multi-dimensional damped
 * exponential moving average that produces the layer input X' = CEMA(X)
 * (Gecko digest, background section on the exponential moving average;
 * paperlayer.ai summary, section 2.1 and Appendix B.1):
 *   u_t[d, j] = beta[d, j] x_t[d]                               (j < h = 16)
 *   h_t[d, j] = alpha u_t + (1 - alpha delta)(cos theta + i sin theta) h_{t-1}
 *   y_t[d]    = Re(sum_j eta[d, j] h_t[d, j])
 * A document start at token t (reset) drops the second term: h_t = alpha u_t.
 * The expansion by beta and the projection by eta are the plainest readings
 * of the pages' "expands each input dimension into h dimensions" and
 * "projected back to a one-dimensional output"; no skip term is added.
 *
 *   x, y          : [B, L, D] dtype `dtype` (device); y may equal x.
 *   alpha, delta, theta, beta : [D, h] fp32 (device), as they enter the
 *                   recurrence (alpha, delta in (0, 1]).
 *   eta           : [D, h, 2] fp32 (device), real and imaginary parts.
 *   reset         : [B, L] uint8 (device) or NULL; non-zero = a document
 *                   starts at that token.
 *   state_in      : [B, D, h, 2] fp32 (device) h_{-1}, or NULL for zero.
 *   state_out     : [B, D, h, 2] fp32 (device) receives h_{L-1}, or NULL; may
 *                   equal state_in.  Chaining state_out into state_in runs a
 *                   long sequence in segments.
 *   h must be 16.  Requires B <= 65535 and L <= 65535 * 256; every pointer
 *   16-byte aligned.
 *
 * Ownership: a per-device workspace of 2 * B * ceil(L / 256) * D * h complex
 * fp32 (chunk states), grown on demand on `stream` and freed by
 * gecko_release().  Asynchronous on `stream`; argument errors are detected on
 * the host before anything is launched.  Returns GECKO_OK, GECKO_ERR_ARG,
 * GECKO_ERR_SHAPE, GECKO_ERR_ALIGN, GECKO_ERR_ALLOC or GECKO_ERR_CUDA.
 */
int gecko_cema_forward(const void* x, void* y, const float* alpha, const float* delta,
                       const float* theta, const float* beta, const float* eta,
                       const uint8_t* reset, const float* state_in, float* state_out,
                       int64_t B, int64_t L, int64_t D, int64_t h, int dtype, void* stream);

/*
 * gecko_tdnorm_forward - timestep decay normalisation, the normalisation
 * before the projections (Gecko digest, section on technical novelty: the
 * decayed mean m_t = beta1 m_{t-1} + (1 - beta1) mu_t with Adam-style bias
 * correction; paperlayer.ai summary, sections 2.2 and 3.1).  Per batch b,
 * token t and group g of D / G contiguous features:
 *   mu_t, s2_t = mean and biased variance of x_t over the group
 *   m_t = beta1 m_{t-1} + (1 - beta1) mu_t,  v_t = beta2 v_{t-1} + (1 - beta2) s2_t
 *   y_t = (x_t - m_t / (1 - beta1^t)) / sqrt(v_t / (1 - beta2^t) + eps) * gamma + bias
 * (t from 1).  The pages print the mean update only; the variance update
 * with beta2, the per-timestep group statistics and the per-feature affine
 * are the plainest readings.
 *
 *   x, y        : [B, L, D] dtype `dtype` (device); y may equal x.
 *   gamma, bias : [D] fp32 (device).
 *   Requires D / G to be a whole multiple of 8, 0 <= beta1, beta2 < 1,
 *   eps >= 0; every pointer 16-byte aligned.
 * Workspace: 4 * B * L * G floats per device, grown on `stream`, freed by
 * gecko_release().  Asynchronous on `stream`; argument errors are found on
 * the host.  Returns GECKO_OK, GECKO_ERR_ARG, GECKO_ERR_SHAPE,
 * GECKO_ERR_ALIGN, GECKO_ERR_ALLOC or GECKO_ERR_CUDA.
 */
int gecko_tdnorm_forward(const void* x, void* y, const float* gamma, const float* bias,
                         int64_t B, int64_t L, int64_t D, int64_t G,
                         float beta1, float beta2, float eps, int dtype, void* stream);

/*
 * Context parallelism: one sequence split into P consecutive segments of
 * T tokens each (one per rank, T % c == 0), run so that the outputs equal a
 * single call over the whole sequence (up to rounding).  The AWM carry is
 * affine in the state once log z is known (Gecko digest, method step
 * details, step 4: M'_{s+1} = A_s M'_s + b_s with A_s = diag(r_s) -
 * diag(rho_s) C~_s), and log z is a prefix of exp-sums (core method), so a
 * rank needs from the ranks before it only their log-exp-sums and their
 * composed segment maps; SCA needs the previous segment's last chunk of K
 * and V (step 3).  A rank r:
 *   1. gecko_awm_segment_logsum(km_r) -> lsum_r; all-gather lsum (P x [B,H,d]);
 *   2. gecko_awm_cp_logz(lsum_all, P, r) -> logz_in_r;
 *      gecko_awm_segment_maps(km_r, v_r, logz_in_r) -> maps_r; all-gather maps;
 *   3. gecko_awm_cp_state(lsum_all, maps_all, P, r) -> state_in_r, then
 *      gecko_sca_awm_forward_continue with k, v prefixed by the previous
 *      segment's last c rows (rank 0: a fresh gecko_sca_awm_forward).
 * All buffers are device memory, fp32 unless stated, 16-byte aligned.
 * gecko_awm_segment_logsum and gecko_awm_segment_maps work in the forward's
 * per-device workspace: after either, gecko_awm_state returns
 * GECKO_ERR_NO_STATE until the next gecko_sca_awm_forward(_continue).
 */
/* lsum_out [B,H,d]: log sum over the segment's tokens of exp(km) per feature.
 * km [B,H,T,d] dtype.  Same size rules and errors as the forward. */
int gecko_awm_segment_logsum(const void* km, float* lsum_out,
                             int64_t B, int64_t H, int64_t T, int64_t c, int64_t d,
                             int dtype, void* stream);
/* maps_out [B,H,4,d,d] = (A, b, A', b'): with log z entering the segment at
 * logz_in [B,H,d] (-inf entries for the first segment), the segment maps its
 * incoming state M'_in to M'_out = A M'_in + b (after its last chunk) and
 * to A' M'_in + b' (before its last chunk).  km, v [B,H,T,d] dtype. */
int gecko_awm_segment_maps(const void* km, const void* v, const float* logz_in, float* maps_out,
                           int64_t B, int64_t H, int64_t T, int64_t c, int64_t d,
                           int dtype, void* stream);
/* logz_out [B,H,d] = logsumexp over the segments j < rank of lsum_all[j]
 * (lsum_all [P,B,H,d]); -inf for rank 0. */
int gecko_awm_cp_logz(const float* lsum_all, int P, int rank, float* logz_out,
                      int64_t B, int64_t H, int64_t d, void* stream);
/* state_out [B,H,2d^2+d] = (M'_prev, M'_in, log z) for segment `rank`, the
 * state_in of gecko_sca_awm_forward_continue, from every rank's lsum
 * [P,B,H,d] and maps [P,B,H,4,d,d] (zeros and -inf for rank 0). */
int gecko_awm_cp_state(const float* lsum_all, const float* maps_all, int P, int rank, float* state_out,
                       int64_t B, int64_t H, int64_t d, void* stream);

/* Thread-local message describing the last non-zero status of this thread. */
const char* gecko_last_error(void);

/* Free the workspace of every device the library used.  Not thread-safe
 * against a concurrent forward. */
void gecko_release(void);

#ifdef __cplusplus
}
#endif

#endif /* GECKO_H */
