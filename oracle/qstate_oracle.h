/*
 * Plain CPU oracle for the quantized recurrent-state decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this code.  The product (the CUDA
 * library under ssm_decode_step_b200/) never calls it and shares no code,
 * header, table or helper with it.
 *
 * What it computes: one decode step of the linear recurrence of
 * "LinQuant: Functional Invariances for Low-Precision Linear Recurrences",
 * Theoretical Foundation, eq. (1):
 *
 *     S_t = S_{t-1} Lambda_t (I - delta beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *
 * with readout o_t = S_t q_t (same page, Low-Precision Chunkwise Realization,
 * "state read"), where the state S (Dv x Dk per tile) is stored as group-wise
 * INT4/INT8 codes plus FP32 scales and is requantized after every step
 * ("When Dynamic Scaling Fails", abstract: the quantizer sits inside the
 * recurrence).  Scale policies: per-token dynamic, persistent, yoked
 * (project page of "When Dynamic Scaling Fails", the feedback-loop section);
 * rounding: nearest or Bounded Directional Rounding ("Preserving Updates in
 * Low-Bit Recurrent State Quantization", abstract).
 *
 * Arithmetic is IEEE FP32 in a fixed operation order (compiled with
 * -ffp-contract=off; fmaf only where written).  The dequantized, decayed
 * state is c * (s * a) (the decay folded into the group scale first).  Dot
 * products are fixed as: per 32-column chunk, eight fused multiply-add
 * chains from +0, chain r over the columns r, r + 8, r + 16, r + 24 of the
 * chunk in that order, chunk sum ((p0 + p4) + (p2 + p6)) + ((p1 + p5) +
 * (p3 + p7)); chunk sums combined by a balanced pairwise tree in column
 * order.
 *
 * Parity status: every function here is pinned by the CPU tests in
 * tests/test_oracle_pins.py (closed forms, invariants, brute force); the
 * whole quantized trajectory has no printed worked example on the pages.
 */
#ifndef QSTATE_ORACLE_H
#define QSTATE_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { QO_DECAY_SCALAR = 0, QO_DECAY_DIAGONAL = 1 };
enum { QO_SCALE_DYNAMIC = 0, QO_SCALE_PERSISTENT = 1, QO_SCALE_YOKED = 2 };
enum { QO_ROUND_NEAREST = 0, QO_ROUND_BDR = 1 };

typedef struct {
  int32_t tiles;    /* independent (layer, batch, head) states            */
  int32_t dk, dv;   /* key and value dimensions; dk = 32 * 2^m            */
  int32_t qmax;     /* largest code magnitude: 2^(bits-1) - 1             */
  int32_t group;    /* quantization group length along dk; divides dk     */
  int32_t delta;    /* 0 = linear write, 1 = delta-rule correction        */
  int32_t decay;    /* QO_DECAY_*                                         */
  int32_t policy;   /* QO_SCALE_*                                         */
  int32_t rounding; /* QO_ROUND_*                                         */
} qo_cfg;

/* Returns 0 when the configuration is one the oracle evaluates, else -1. */
int qo_check(const qo_cfg* c);

/* Number of OpenMP threads the tile loops use. */
int qo_num_threads(void);

/* Codes are kept unpacked here, one int32 per element, [tiles][dv][dk];
 * qo_pack / qo_unpack convert to the packed byte layout (INT8: one byte per
 * element; INT4: two per byte, even column in the low nibble), both in
 * two's complement. */
int qo_pack(int bits, int64_t n, const int32_t* codes, uint8_t* packed);
int qo_unpack(int bits, int64_t n, const uint8_t* packed, int32_t* codes);

/* Quantization start: per (row, group) scale = max|S0| / qmax, codes by
 * nearest rounding; the yoked shadow (if non-NULL) becomes a copy of S0. */
int qo_init(const qo_cfg* c, const float* S0, int32_t* codes, float* scales,
            float* shadow);

/* One decode step in place on (codes, scales, shadow).  q, k: [tiles][dk];
 * v: [tiles][dv]; alpha: [tiles] (scalar) or [tiles][dk] (diagonal);
 * beta: [tiles]; o: [tiles][dv] or NULL.  prequant (optional,
 * [tiles][dv][dk] doubles) receives the exact pre-rounding value x * inv of
 * every element, NaN for zero-scale groups. */
int qo_step(const qo_cfg* c, int32_t* codes, float* scales, float* shadow,
            const float* q, const float* k, const float* v,
            const float* alpha, const float* beta, float* o,
            double* prequant);

/* Low-Rank Bypass ("Preserving Updates in Low-Bit Recurrent State
 * Quantization", abstract: small updates accumulate in a compact low-rank
 * buffer that is periodically merged into the state).  Reading taken here:
 * the buffer holds the last writes of the current period as rank-1 terms
 * w k^T in FP32 (U [tiles][dv][rank], keys K [tiles][rank][dk] decayed in
 * place), and the stored codes are not touched between merges; their decay
 * accumulates per column in A [tiles][dk].  The period is `rank` steps; slot
 * = position of this step in it (0 .. rank-1).  Per tile:
 *   a. A_j = (slot ? A_in_j : 1) * a_j;  K'_r = K_in_r * a (r < slot)
 *   b. kk_r = K'_r . k, kq_r = K'_r . q, kqn = k . q
 *   c. S'_ij = c_ij * (s_ig * A_j)
 *   d. u_i = S'_i . k, then u_i = fused(U_ri * kk_r + u_i) for r < slot;
 *      w_i = beta (v_i - u_i) (delta 1) or beta v_i
 *   e. slot < rank-1 (bypass): o_i = S'_i . q, then fused(U_ir kq_r + o_i)
 *      for r < slot, then fused(w_i kqn + o_i); U_i,slot = w_i; A_out = A,
 *      K_out_r = K'_r (r < slot), K_out_slot = k; codes and scales kept
 *   f. slot = rank-1 (merge): x_ij = S'_ij, then fused(U_ri K'_rj + x_ij)
 *      for r < slot, then fused(w_i k_j + x_ij); o_i = x_i . q; requantize x
 *      as qo_step does, with BDR's sigma_ij = sign(M_ij), M_ij the same
 *      chain from +0 (the accumulated update), and its reference the stored
 *      element c_ij * s_ig.
 * The yoked shadow advances by qo_step's rule at every step.  With rank 1
 * every step is a merge and the step is qo_step's.  A_out, K_out may be NULL
 * at a merge; A_in, K_in may be NULL at slot 0. */
int qo_lrb_step(const qo_cfg* c, int rank, int slot, int32_t* codes, float* scales,
                float* shadow, const float* A_in, float* A_out, const float* K_in,
                float* K_out, float* U, const float* q, const float* k, const float* v,
                const float* alpha, const float* beta, float* o, double* prequant);

/* o = dequant(S) q with the state unchanged. */
int qo_readout(const qo_cfg* c, const int32_t* codes, const float* scales,
               const float* q, float* o);

/* The unquantized FP32 recurrence, in place on S [tiles][dv][dk], in the
 * same operation order as the quantized step (this is also the yoked
 * shadow's update).  o may be NULL. */
int qo_fp32_step(const qo_cfg* c, float* S, const float* q, const float* k,
                 const float* v, const float* alpha, const float* beta,
                 float* o);

/* Squared Frobenius norm of each tile, out[t] (doubles), summed in FP64 in
 * row-major order: of the dequantized stored state (d = c * s in FP32, as in
 * qo_readout), and of an FP32 state [tiles][dv][dk].  The state norm over a
 * decode horizon is the quantity whose inflation under per-token dynamic
 * scaling "When Dynamic Scaling Fails" reports (abstract, project page). */
int qo_sq_norms(const qo_cfg* c, const int32_t* codes, const float* scales, double* out);
int qo_fp32_sq_norms(const qo_cfg* c, const float* S, double* out);

/* The fixed-order dot product used throughout (exposed for tests). */
float qo_dot(const float* a, const float* b, int n);

/* Mistakes that a mutation test plants on purpose, to show that the pins
 * catch them.  Only the mutation build of this file (compiled with
 * QO_MUTATIONS into liboracle_mut.so) has them and exports qo_set_fault;
 * the oracle proper (liboracle.so) is compiled without them. */
enum {
  QO_FAULT_NONE = 0,
  QO_FAULT_DROP_DELTA = 1,      /* delta-rule correction term left out       */
  QO_FAULT_WRITE_SIGN = 2,      /* write term added with the wrong sign      */
  QO_FAULT_DECAY_SKIPPED = 3,   /* decay not applied                         */
  QO_FAULT_READ_K_FOR_Q = 4,    /* readout uses k instead of q               */
  QO_FAULT_GROUP_INDEX = 5,     /* scale of the wrong group used             */
  QO_FAULT_BDR_REFERENCE = 6,   /* BDR measured from the decayed value S'    */
  QO_FAULT_ROUND_TRUNC = 7,     /* truncation instead of nearest rounding    */
  QO_FAULT_BETA_ON_V_ONLY = 8,  /* beta applied to v but not to the delta term */
  QO_FAULT_DIAG_DECAY_ROW = 9,  /* diagonal decay indexed by row, not column  */
  QO_FAULT_PERSIST_UPDATE = 10, /* persistent scale recomputed every step    */
  QO_FAULT_YOKED_FROM_X = 11,   /* yoked scale taken from the quantized path */
  QO_FAULT_LRB_SIGN_LAST = 12,  /* merge BDR sign from the last write only   */
  QO_FAULT_COUNT = 13
};
#ifdef QO_MUTATIONS
void qo_set_fault(int fault);
#endif

#ifdef __cplusplus
}
#endif
#endif
