/*
 * qstate — quantized recurrent-state decode step for NVIDIA B200 (sm_100a).
 *
 * One decode step of the linear recurrence of "LinQuant: Functional
 * Invariances for Low-Precision Linear Recurrences" (Theoretical
 * Foundation, eq. (1)):
 *
 *     S_t = S_{t-1} Lambda_t (I - delta beta_t k_t k_t^T) + beta_t v_t k_t^T
 *
 * with readout o_t = S_t q_t (same page, Low-Precision Chunkwise
 * Realization, "state read").  S is a Dv x Dk matrix per tile, one tile
 * per (layer, batch, head); tiles are independent.  The state lives in
 * device memory as group-wise INT4 or INT8 codes plus one FP32 scale per
 * group of `group` consecutive columns of a row, and every step
 * dequantizes, decays, writes, reads out and requantizes it in one pass
 * (a quantizer applied inside the recurrence: "When Dynamic Scaling
 * Fails", abstract).
 *
 * Element-level definition (FP32, IEEE round to nearest even; "fused"
 * means one rounding), for tile t, row i, column j, group g = j / group:
 *   S'_ij = c_ij * (s_ig * a_j)              dequantized previous state with
 *                                            the decay folded into the scale:
 *                                            a_j = alpha_t (QS_DECAY_SCALAR)
 *                                            or alpha_tj (QS_DECAY_DIAGONAL)
 *   w_i   = beta_t * (v_i - u_i), u_i = S'_i . k   (delta = 1)
 *   w_i   = beta_t * v_i                           (delta = 0)
 *   x_ij  = fused(w_i * k_j + S'_ij)         updated state
 *   o_i   = x_i . q                          readout, before requantization
 *   s'_ig = max_{j in g} |x_ij| / qmax       QS_SCALE_DYNAMIC
 *         = s_ig                             QS_SCALE_PERSISTENT
 *         = max_{j in g} |R_ij| / qmax       QS_SCALE_YOKED, R = FP32 shadow
 *                                            updated by the same steps
 *   if s'_ig > 0: n_ij = clamp(round_half_even(x_ij * (1/s'_ig)), +-qmax),
 *                 the product taken exactly; else n_ij = 0 for the group
 *   BDR: with sigma = sign(w_i) sign(k_j) and d_ij = c_ij * s_ig the
 *        element as stored before the step (no decay), if sigma > 0 and
 *        n s' < d_ij then n += 1; if sigma < 0 and n s' > d_ij then
 *        n -= 1; clamp.  ("Preserving Updates in Low-Bit Recurrent State
 *        Quantization", abstract: a stored element whose value moves
 *        against its update is rounded one step toward it.)
 * qmax = 2^(bits-1) - 1.  Dot products "." are evaluated in one fixed
 * order: each 32-column chunk is summed as eight fused multiply-add chains
 * from +0, chain r over the chunk's columns r, r+8, r+16, r+24 in that
 * order; the chunk sum is ((p0 + p4) + (p2 + p6)) + ((p1 + p5) + (p3 + p7));
 * and the chunk sums are combined by a balanced pairwise tree in column
 * order.  Codes, scales and the shadow are therefore reproducible bit for
 * bit on any conforming implementation.
 *
 * Scale policies ("When Dynamic Scaling Fails", project page): per-token
 * dynamic reads its scale from the state it is about to quantize;
 * persistent fixes the scale at the quantization start (qstate_init) and
 * clips; yoked takes it from a full-precision reference run alongside.
 *
 * Memory layout (all row-major, tile-major, no padding):
 *   codes   [T][Dv][Dk*bits/8] bytes, two's complement; INT4 packs the even
 *           column in the low nibble of each byte
 *   scales  [T][Dv][Dk/group]  float
 *   shadow  [T][Dv][Dk]        float   (QS_SCALE_YOKED only)
 *   q, k    [T][Dk]            float
 *   v       [T][Dv]            float
 *   alpha   [T] (scalar decay) or [T][Dk] (diagonal decay)  float
 *   beta    [T]                float
 *   o       [T][Dv]            float
 *
 * Conventions for every entry point:
 *   - All array pointers are DEVICE pointers owned by the caller; the
 *     library allocates no memory and keeps no state between calls (the
 *     host-buffer pipeline below is the one exception: it owns its staging
 *     buffers, streams and events).
 *   - codes, scales, shadow are updated in place; other inputs are read.
 *   - Work is enqueued on `stream` and returns immediately; QS_OK means
 *     "validated and launched".  Execution errors surface at the caller's
 *     next synchronization on that stream.
 *   - Stream order holds as for any launch.  The decode-step, readout and
 *     FP32-step kernels are launched with programmatic dependent launch:
 *     they may be scheduled while the kernel before them in the stream
 *     finishes, and wait for it to complete (its writes visible) before
 *     touching any memory.  The environment variable QSTATE_PDL=0 launches
 *     them plainly.
 *   - Arguments are validated before anything is launched.  A NULL
 *     required pointer, a misaligned pointer (codes, shadow: 32 bytes;
 *     S0, scales, q, k, v, alpha when diagonal: 16 bytes; alpha when
 *     scalar, beta, o: 4 bytes), overlapping buffers, or an out-of-range field
 *     returns QS_ERR_INVALID_ARG; a valid configuration this build has no
 *     kernel for returns QS_ERR_UNSUPPORTED; a failed launch returns
 *     QS_ERR_CUDA.  Nothing aborts or throws across this boundary.
 *   - Values: beta > 0 and |Lambda| <= 1 are the caller's contract and are
 *     not checked.  Non-finite inputs give unspecified codes but every
 *     access stays in bounds.
 *   - Calls that overlap on the GPU must not share state buffers.
 *
 * Supported by this build: dk in {64, 128}; dv a multiple of 16 with
 * 16 <= dv <= 4096; bits in {4, 8}; group in {32, 64, 128} with
 * group <= dk; num_tiles >= 0 with num_tiles * dv / 8 < 2^31.
 */
#ifndef QSTATE_H
#define QSTATE_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define QS_API __attribute__((visibility("default")))
#else
#define QS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QS_OK = 0,
  QS_ERR_INVALID_ARG = 1,
  QS_ERR_UNSUPPORTED = 2,
  QS_ERR_CUDA = 3
} qs_status;

typedef enum { QS_DECAY_SCALAR = 0, QS_DECAY_DIAGONAL = 1 } qs_decay;
typedef enum {
  QS_SCALE_DYNAMIC = 0,
  QS_SCALE_PERSISTENT = 1,
  QS_SCALE_YOKED = 2
} qs_policy;
typedef enum { QS_ROUND_NEAREST = 0, QS_ROUND_BDR = 1 } qs_rounding;

/* Configuration of one family of states (eq. (1) choices + storage).
 * Fixed-width fields so the layout is the same from any language. */
typedef struct {
  int32_t num_tiles; /* layers * batch * heads; tiles are independent      */
  int32_t dk;        /* key dimension (columns of S)                      */
  int32_t dv;        /* value dimension (rows of S)                       */
  int32_t bits;      /* 4 or 8                                            */
  int32_t group;     /* quantization group length along dk                */
  int32_t delta;     /* 0: linear write; 1: delta-rule correction         */
  int32_t decay;     /* qs_decay: Lambda = alpha I or diag(alpha)          */
  int32_t policy;    /* qs_policy                                          */
  int32_t rounding;  /* qs_rounding                                        */
} qs_config;

/* Bytes of each state buffer for `cfg` (shadow_bytes is 0 unless yoked).
 * Any of the output pointers may be NULL.  Host-only; launches nothing. */
QS_API qs_status qstate_query_sizes(const qs_config* cfg, size_t* codes_bytes,
                             size_t* scales_bytes, size_t* shadow_bytes);

/* Quantization start: from the FP32 state S0 [T][Dv][Dk] (device), write
 * codes and scales with the dynamic rule (scale = group max|S0| / qmax,
 * nearest rounding) — under QS_SCALE_PERSISTENT these scales stay fixed
 * from here on — and, for QS_SCALE_YOKED, copy S0 into the shadow.
 * shadow is ignored (may be NULL) for the other policies. */
QS_API qs_status qstate_init(const qs_config* cfg, const float* S0, void* codes,
                      float* scales, float* shadow, cudaStream_t stream);

/* One decode step, in place on (codes, scales, shadow), as defined above.
 * q may be NULL only when o is NULL; o == NULL skips the readout.
 * alpha is [T] for QS_DECAY_SCALAR and [T][Dk] for QS_DECAY_DIAGONAL. */
QS_API qs_status qstate_decode_step(const qs_config* cfg, void* codes, float* scales,
                             float* shadow, const float* q, const float* k,
                             const float* v, const float* alpha,
                             const float* beta, float* o, cudaStream_t stream);

/* Host-buffer decode pipeline: one decode step per call, as
 * qstate_decode_step defines it, of n state families (at most 8) that
 * consume the same token's inputs, with the inputs read from HOST memory
 * and the readouts written back to HOST memory.  The pipeline owns `depth`
 * (2..8) device copies of one step's inputs and readouts, a copy-in
 * stream, a copy-out stream and their events: step t's inputs go up on the
 * copy-in stream while earlier steps compute, its state updates run on the
 * caller's stream (in call order), and its readouts come down on the
 * copy-out stream while later steps compute.
 *
 * Host input of one step (packed, float): q [T][Dk] | k [T][Dk] | v [T][Dv]
 * | alpha [T] (scalar decay) or [T][Dk] (diagonal) | beta [T].  Host output
 * of one step: o [n][T][Dv] (family i's readout at offset i*T*Dv).  Page-
 * locked host memory makes the copies asynchronous.  The copies of step t
 * are in flight after the call returns: the caller keeps step t's input
 * unchanged and does not read its output until qstate_pipeline_sync has
 * returned, or until the call for step t + depth has returned (each call
 * first waits, on the host, for the copies of the step that last used its
 * device buffers).
 *
 * All families share num_tiles, dk, dv, delta and decay (each passes
 * qstate_decode_step's checks); they differ in bits, group, policy and
 * rounding.  The pipeline belongs to the device current at creation; calls
 * from another current device return QS_ERR_INVALID_ARG.  One host thread
 * at a time may use a pipeline.  After an error
 * from qstate_pipeline_step the pipeline may hold a partial step: sync and
 * destroy it. */
typedef struct qs_pipeline qs_pipeline;

/* Bytes of one step's host input and host output for n families of cfg.
 * Host-only; launches nothing. */
QS_API qs_status qstate_pipeline_query_sizes(const qs_config* cfg, int n, size_t* in_bytes,
                                             size_t* out_bytes);

/* Create a pipeline for families cfgs[0..n-1] with `depth` buffers on the
 * current device (device memory, two streams, events).  Arguments are
 * checked before any CUDA call. */
QS_API qs_status qstate_pipeline_create(int n, const qs_config* cfgs, int depth,
                                        qs_pipeline** out);

/* Issue one step.  codes[i], scales[i], shadow[i]: family i's state (as for
 * qstate_decode_step; shadow may be NULL, or shadow[i] NULL, for families
 * that are not yoked).  host_out == NULL skips the readouts (no output
 * copy).  `stream` runs the state updates. */
QS_API qs_status qstate_pipeline_step(qs_pipeline* pl, void* const* codes, float* const* scales,
                                      float* const* shadow, const void* host_in, void* host_out,
                                      cudaStream_t stream);

/* Make the pipeline's copy streams wait for the work submitted to `stream`
 * so far (e.g. an event that opens a timed region), without blocking the
 * host. */
QS_API qs_status qstate_pipeline_wait_stream(qs_pipeline* pl, cudaStream_t stream);

/* Make `stream` wait for every copy the pipeline has issued, without
 * blocking the host. */
QS_API qs_status qstate_pipeline_join(qs_pipeline* pl, cudaStream_t stream);

/* Block the host until every step issued so far, with its copies, is done. */
QS_API qs_status qstate_pipeline_sync(qs_pipeline* pl);

/* Synchronize, then free the pipeline's device memory, streams and events.
 * NULL is accepted and ignored. */
QS_API qs_status qstate_pipeline_destroy(qs_pipeline* pl);

/* Bytes of device memory that qstate_decode_step_host_static stages one
 * step through (32 MiB): a static array of the library that every GPU which
 * loads the library holds until the process exits. */
#define QS_STATIC_STAGE_BYTES ((size_t)32 << 20)

/* One decode step of one state family, as qstate_decode_step defines it,
 * with its inputs read from HOST memory and its readouts written back to
 * HOST memory, that allocates nothing.  It has no counterpart in the pages
 * the method comes from: it exists for callers that may not allocate device
 * memory themselves, such as an engine whose own memory manager owns the
 * whole device budget (a cudaMalloc outside it can fail or fragment that
 * budget) or a serving loop that cannot afford cudaMalloc's implicit
 * device-wide synchronization.  The host-buffer pipeline above stages
 * through device buffers it allocates at creation; this call stages through
 * a fixed static device array of QS_STATIC_STAGE_BYTES bytes instead, and
 * calls no cudaMalloc, cudaFree or other allocating routine.
 *
 * host_in: the packed host input of one step in the pipeline's layout
 * (q | k | v | alpha | beta, qstate_pipeline_query_sizes with n = 1);
 * host_out: o [T][Dv] floats, or NULL for no readout.  codes, scales and
 * shadow are DEVICE pointers, as for qstate_decode_step.  Everything is
 * enqueued on `stream` in order: the input copy, the step, the output copy;
 * the caller keeps host_in unchanged and reads host_out only after
 * synchronizing with `stream`.  Page-locked host memory makes the copies
 * asynchronous.
 *
 * Limits and sharing: a step whose input bytes plus (when host_out is not
 * NULL) output bytes exceed QS_STATIC_STAGE_BYTES returns
 * QS_ERR_UNSUPPORTED before any CUDA call.  The first call on a device looks
 * up the array's device address on that device (with it current) and keeps
 * it; make that first call before any stream capture.  Every call on a
 * device shares the one array, which keeps the last call's contents: each
 * call writes every byte it reads from it, so nothing needs to start at
 * zero, but calls that overlap on the GPU (on different streams, or from
 * several host threads) overwrite each other's staging and race.  The other
 * argument checks and errors are qstate_decode_step's. */
QS_API qs_status qstate_decode_step_host_static(const qs_config* cfg, void* codes, float* scales,
                                                float* shadow, const void* host_in, float* host_out,
                                                cudaStream_t stream);

/* Readout of the stored state without changing it: o_i = d_i . q with
 * d_ij = c_ij * s_ig (no decay; the fixed dot order above). */
QS_API qs_status qstate_readout(const qs_config* cfg, const void* codes,
                         const float* scales, const float* q, float* o,
                         cudaStream_t stream);

/* One decode step of the UNQUANTIZED recurrence (the same definition with
 * the state kept in FP32: the baseline "FP32 state" the quantized state is
 * measured against).  S [T][Dv][Dk] float, 32-byte aligned, updated in
 * place: S <- (S * a) + w k^T with w as above (same fixed order); readout
 * o = S_t q (o == NULL skips it; q may then be NULL).  Only num_tiles, dk,
 * dv, delta and decay of cfg are used. */
QS_API qs_status qstate_fp32_decode_step(const qs_config* cfg, float* S, const float* q,
                                         const float* k, const float* v, const float* alpha,
                                         const float* beta, float* o, cudaStream_t stream);

/* Low-Rank Bypass ("Preserving Updates in Low-Bit Recurrent State
 * Quantization", abstract: small updates are accumulated in a compact
 * low-rank buffer whose elements are periodically merged into the state).
 * Reading implemented here: over a period of `rank` steps the writes w k^T
 * bypass the quantized state and are held in FP32 as rank-1 terms; the
 * stored codes and scales are not touched between merges and their decay
 * accumulates per column; the last step of the period merges the buffer
 * into the state and requantizes it once with the configured scale policy
 * and rounding.  Per tile, for the step at position `slot` of the period:
 *   A_j    = (slot ? A_in_j : 1) * a_j;   K'_r = K_in_r * a   (r < slot)
 *   kk_r   = K'_r . k,  kq_r = K'_r . q,  kqn = k . q
 *   S'_ij  = c_ij * (s_ig * A_j)
 *   u_i    = S'_i . k, then fused(U_ir * kk_r + u_i) for r < slot (delta 1)
 *   w_i    = beta (v_i - u_i)  or  beta v_i
 *   bypass (slot < rank-1): o_i = S'_i . q, fused(U_ir kq_r + o_i) for
 *          r < slot, fused(w_i kqn + o_i); U_i,slot = w_i; A_out = A;
 *          K_out_r = K'_r (r < slot), K_out_slot = k; codes, scales kept
 *   merge  (slot = rank-1): x_ij = S'_ij, fused(U_ir K'_rj + x_ij) for
 *          r < slot, fused(w_i k_j + x_ij); o_i = x_i . q; x is requantized
 *          as by qstate_decode_step, with BDR's sigma_ij = sign(M_ij), M_ij
 *          the same chain started from +0 (the update accumulated over the
 *          period), and its reference the stored element c_ij * s_ig
 * The yoked shadow advances by qstate_decode_step's rule at every step.
 * rank 1 makes every step a merge: the step is then qstate_decode_step's
 * (and is dispatched to it; no buffer is used).
 * Buffers (the caller's, 16-byte aligned; sizes from qstate_lrb_query_sizes):
 *   A_in, A_out [T][Dk] float   accumulated column decay (two copies: read
 *                               one, write the other; A_in unused at slot 0,
 *                               A_out unused at the merge; under scalar decay
 *                               every column holds the same value, as the
 *                               library writes it, and column 0 is read)
 *   K_in, K_out [T][rank][Dk]   buffered keys, decayed (same two copies)
 *   U           [T][Dv][rpad]   buffered write coefficients, rpad = rank
 *                               rounded up to a multiple of 4; column slot is
 *                               written at bypass steps, columns < slot read
 * Supported: 1 <= rank <= 16, 0 <= slot < rank; other fields as for
 * qstate_decode_step.  The caller advances slot (0, 1, ..., rank-1, 0, ...)
 * and swaps the A and K copies after every bypass step. */
QS_API qs_status qstate_lrb_query_sizes(const qs_config* cfg, int rank, size_t* decay_bytes,
                                        size_t* keys_bytes, size_t* coef_bytes);
QS_API qs_status qstate_lrb_decode_step(const qs_config* cfg, int rank, int slot, void* codes,
                                        float* scales, float* shadow, const float* A_in,
                                        float* A_out, const float* K_in, float* K_out, float* U,
                                        const float* q, const float* k, const float* v,
                                        const float* alpha, const float* beta, float* o,
                                        cudaStream_t stream);

/* Chunkwise prefill of an FP32 state over `length` tokens, for the linear
 * write (delta = 0) with scalar decay (the Mamba-2 family whose chunkwise
 * realization LinQuant gives: Low-Precision Chunkwise Realization, state
 * write / state pass / state read / local score / intra-chunk output) or
 * diagonal decay (the GLA family, the same contractions per channel), and
 * for the delta rule (delta = 1, the DeltaNet / Gated DeltaNet family, with
 * either decay).  It computes, for every tile, the token-by-token recurrence
 * of qstate_decode_step on an FP32 state,
 *   S_t = S_{t-1} Lambda_t (I - delta beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *   o_t = S_t q_t,
 * regrouped in chunks of 32 tokens (under the delta rule the corrected
 * values w_t = beta_t (v_t - S_{t-1} Lambda_t k_t) of a chunk solve a unit
 * lower-triangular system, by forward substitution; exact in real
 * arithmetic; in FP32 the
 * summation order differs from the token-by-token order, so results agree
 * with qstate_fp32_decode_step applied token by token to within FP32
 * rounding, not bit for bit).  The state it leaves is the S0 that
 * qstate_init quantizes for the decode path.
 *   S      [T][Dv][Dk] float, in: state before the first token (e.g. zeros),
 *          out: state after the last
 *   q, k   [T][length][Dk] float;  v [T][length][Dv] float
 *   alpha  [T][length] (QS_DECAY_SCALAR) or [T][length][Dk] (diagonal), in (0, 1]
 *   beta   [T][length] float
 *   o      [T][length][Dv] float, or NULL to skip the outputs
 * Only num_tiles, dk, dv, delta and decay of cfg are used; dv <= 128.
 * Under diagonal decay a chunk may decay a channel by at most e^-170. */
QS_API qs_status qstate_prefill(const qs_config* cfg, int length, float* S, const float* q,
                                const float* k, const float* v, const float* alpha,
                                const float* beta, float* o, cudaStream_t stream);

/* The same prefill with its four contractions on the tensor cores
 * (tcgen05.mma, kind::tf32, FP32 accumulators in tensor memory; chunks of
 * 64 tokens; the state stays in tensor memory for the whole sequence).
 * The operands of every contraction are rounded to TF32 (10 explicit
 * mantissa bits, round to nearest with ties away from zero, as cvt.rna
 * does) and the state is read at TF32 precision (low mantissa bits
 * dropped) by the state read, so results agree with the FP32 recurrence
 * to about 2^-10 of the magnitudes summed, not to FP32 rounding: every
 * element of S and o is within 2^-8 of the same recurrence run on |S0|,
 * |q|, |k|, |v| (the sum of the magnitudes of its terms).  Arguments,
 * validation are those of qstate_prefill, with S, q and k 16-byte aligned
 * and the linear write only (delta = 1 returns QS_ERR_UNSUPPORTED);
 * under either decay a chunk of 64 tokens may decay a channel by at most
 * e^-170 (the decay factors are split around the chunk's middle token).
 * A wait for the tensor cores that does not end (a bounded poll) makes the
 * CTA free its tensor memory and return; qstate_prefill_tf32_timeouts
 * reports the count.  After a launch that counted a timeout, S and o of
 * that launch are undefined: compare the count before and after the call
 * (after synchronizing) and discard the results when it rose. */
QS_API qs_status qstate_prefill_tf32(const qs_config* cfg, int length, float* S, const float* q,
                                     const float* k, const float* v, const float* alpha,
                                     const float* beta, float* o, cudaStream_t stream);

/* Number of CTAs of qstate_prefill_tf32 whose wait for the tensor cores gave
 * up since the library was loaded (current device; synchronous). */
QS_API qs_status qstate_prefill_tf32_timeouts(unsigned int* count);

/* Self-check of that bounded wait: launches one CTA of the tensor-core
 * prefill kernel in a mode whose first wait for the tensor cores cannot
 * complete (nothing has been committed to it), with a limit of `polls`
 * polls; the CTA must give up, count the timeout, free its tensor memory
 * and return, leaving the context usable.  Synchronous on the legacy
 * default stream; *timed_out receives the number of CTAs that reported a
 * timeout (1 when the mechanism works).  polls in [1, 2^20], else
 * QS_ERR_INVALID_ARG before any launch. */
QS_API qs_status qstate_prefill_tf32_wait_selfcheck(unsigned int polls, unsigned int* timed_out);

/* Squared Frobenius norm of every tile of the stored state, for tracking
 * the state norm over a decode horizon (the norm inflation of per-token
 * dynamic scaling: "When Dynamic Scaling Fails", abstract and project page,
 * the feedback-loop passage).  out[t] = sum over (i, j) of d_ij^2 with
 * d_ij = c_ij * s_ig formed in FP32 as in qstate_readout, each square and
 * the sum in FP64 (summation order unspecified: the result is the exact
 * sum up to FP64 rounding).  out: device array of num_tiles doubles,
 * 8-byte aligned, written on `stream`. */
QS_API qs_status qstate_state_sq_norms(const qs_config* cfg, const void* codes,
                                       const float* scales, double* out, cudaStream_t stream);

/* The same for an FP32 state S [T][Dv][Dk] (16-byte aligned): out[t] = sum
 * of S_ij^2 in FP64.  Only num_tiles, dk and dv of cfg are used. */
QS_API qs_status qstate_fp32_sq_norms(const qs_config* cfg, const float* S, double* out,
                                      cudaStream_t stream);

/* Self-check of the library's fast arithmetic on the current GPU.  The
 * kernels compute the reciprocal of a scale and the division of a group
 * maximum by qmax with short fused multiply-add sequences; this compares
 * them bit for bit with the IEEE correctly rounded results on every input:
 * the reciprocal on every float in [2^-126, 2^126), the divisions by 7 and
 * by 127 on every finite non-negative float (about 6.4e9 evaluations).
 * mismatches: device array of 3 unsigned 64-bit counters (reciprocal, /7,
 * /127), 8-byte aligned, zeroed and filled on `stream`.  All three must be
 * 0; the caller reads them after synchronizing. */
QS_API qs_status qstate_selfcheck(unsigned long long* mismatches, cudaStream_t stream);

/* Static, human-readable name of a status code. */
QS_API const char* qstate_status_string(qs_status status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
QS_API int qstate_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QSTATE_H */
