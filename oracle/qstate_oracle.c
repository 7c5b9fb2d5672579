/*
 * Plain CPU oracle for the quantized recurrent-state decode step.
 * TEST INFRASTRUCTURE ONLY (see qstate_oracle.h): nothing in the product
 * calls this file.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -fopenmp -fPIC -shared
 * (oracle/build.py).  All arithmetic is IEEE FP32; fmaf appears exactly
 * where the operation order below says "fused".
 *
 * Element-level definition followed here, per tile and row i:
 *   1. dequantize and decay   S'_j = c_ij * (s_ig * a_j)   (decayed scale)
 *        (a_j = alpha for scalar decay Lambda = alpha I, alpha_j for
 *         Lambda = diag(alpha): LinQuant, Key structural choices)
 *   2. write coefficient      w = beta * (v_i - u)   with u = S' . k  (delta 1)
 *                             w = beta * v_i                          (delta 0)
 *        eq. (1) rearranged: S'(I - beta k k^T) + beta v k^T = S' + (beta (v - S'k)) k^T
 *   3. rank-1 write           x_j = fused(w * k_j + S'_j)
 *   4. readout                o_i = x . q   (updated state, before requantization)
 *   5. yoked shadow           the same steps 1-3 on the FP32 shadow R
 *   6. scale per group        dynamic:    s' = max|x_j| / qmax
 *                             persistent: s' = s (fixed at quantization start)
 *                             yoked:      s' = max|R_j| / qmax
 *   7. rounding               s' not > 0: every code of the group is 0;
 *                             else inv = 1/s', n = nearest integer to the exact
 *                             product x_j * inv (ties to even), clamped to
 *                             [-qmax, qmax]
 *   8. BDR (if selected)      sigma = sign(w) sign(k_j), d_j = c_ij * s_ig
 *                             (the element as stored before the step); if
 *                             sigma > 0 and n*s' < d_j then n += 1; if
 *                             sigma < 0 and n*s' > d_j then n -= 1; clamp
 *   9. store                  codes, and s' for dynamic / yoked
 * Dot products "." use qo_dot's fixed order (eight interleaved chains per
 * 32 entries, pairwise tree over the chunks).
 */
#include "qstate_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define QO_MAX_DK 1024
#define QO_MAX_RANK 32

/* Planted mistakes (test build only).  The oracle proper is compiled
 * without QO_MUTATIONS, where every FAULT(...) below is the constant 0 and
 * the branches it guards are gone; oracle/build.py compiles the same file a
 * second time with QO_MUTATIONS into a separate library that the mutation
 * test alone loads. */
#ifdef QO_MUTATIONS
static int g_fault = QO_FAULT_NONE;
void qo_set_fault(int fault) { g_fault = fault; }
#define FAULT(x) (g_fault == (x))
#else
#define FAULT(x) 0
#endif

int qo_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

int qo_check(const qo_cfg* c) {
  if (!c) return -1;
  if (c->tiles < 0 || c->dv < 1) return -1;
  if (c->dk < 32 || c->dk > QO_MAX_DK || c->dk % 32) return -1;
  int chunks = c->dk / 32;
  if (chunks & (chunks - 1)) return -1;
  if (c->qmax < 1 || c->qmax > (1 << 20)) return -1;
  if (c->group < 1 || c->dk % c->group) return -1;
  if (c->delta != 0 && c->delta != 1) return -1;
  if (c->decay != QO_DECAY_SCALAR && c->decay != QO_DECAY_DIAGONAL) return -1;
  if (c->policy < QO_SCALE_DYNAMIC || c->policy > QO_SCALE_YOKED) return -1;
  if (c->rounding != QO_ROUND_NEAREST && c->rounding != QO_ROUND_BDR) return -1;
  return 0;
}

/* Fixed-order dot product over n = 32 * 2^m entries.  Each 32-entry chunk
 * is summed as eight fused multiply-add chains from +0, chain r over the
 * entries j = r, r + 8, r + 16, r + 24 of the chunk in that order; the chunk
 * sum is ((p0 + p4) + (p2 + p6)) + ((p1 + p5) + (p3 + p7)); the chunk sums
 * are combined by a balanced pairwise tree in order: ((c0 + c1) + (c2 + c3))
 * + ... */
float qo_dot(const float* a, const float* b, int n) {
  float part[QO_MAX_DK / 32];
  int chunks = n / 32;
  for (int c = 0; c < chunks; ++c) {
    float p[8];
    for (int r = 0; r < 8; ++r) p[r] = 0.0f;
    for (int j = 0; j < 32; ++j) p[j % 8] = fmaf(a[32 * c + j], b[32 * c + j], p[j % 8]);
    part[c] = ((p[0] + p[4]) + (p[2] + p[6])) + ((p[1] + p[5]) + (p[3] + p[7]));
  }
  for (int width = chunks; width > 1; width /= 2)
    for (int m = 0; m < width / 2; ++m) part[m] = part[2 * m] + part[2 * m + 1];
  return part[0];
}

static float sign_of(float x) { return x > 0.0f ? 1.0f : (x < 0.0f ? -1.0f : 0.0f); }

/* Decay factor applied to column j of row i of tile t. */
static float decay_at(const qo_cfg* c, const float* alpha, int t, int i, int j) {
  if (FAULT(QO_FAULT_DECAY_SKIPPED)) return 1.0f;
  if (c->decay == QO_DECAY_SCALAR) return alpha[t];
  if (FAULT(QO_FAULT_DIAG_DECAY_ROW)) return alpha[(size_t)t * c->dk + (i % c->dk)];
  return alpha[(size_t)t * c->dk + j];
}

/* Steps 2-3 for one row: given the decayed row Sp, return w and write the
 * updated row into x.  Shared by the quantized path, the yoked shadow and
 * the unquantized recurrence, so the three see one definition. */
static float row_write(const qo_cfg* c, const float* Sp, const float* k, float v_i,
                       float beta, float* x) {
  const int dk = c->dk;
  float w;
  if (c->delta && !FAULT(QO_FAULT_DROP_DELTA)) {
    float u = qo_dot(Sp, k, dk);
    if (FAULT(QO_FAULT_BETA_ON_V_ONLY))
      w = beta * v_i - u;
    else
      w = beta * (v_i - u);
  } else {
    w = beta * v_i;
  }
  for (int j = 0; j < dk; ++j) {
    if (FAULT(QO_FAULT_WRITE_SIGN))
      x[j] = fmaf(-w, k[j], Sp[j]);
    else
      x[j] = fmaf(w, k[j], Sp[j]);
  }
  return w;
}

/* Step 7: nearest code.  The product of two floats is exact in double
 * (24 + 24 significant bits), so rint gives the nearest integer to the
 * exact product, ties to even.  fmax/fmin return the non-NaN operand, so a
 * NaN product lands on -qmax. */
static int32_t nearest_code(float x, float inv, int qmax, double* pre) {
  double p = (double)x * (double)inv;
  if (pre) *pre = p;
  double r = (FAULT(QO_FAULT_ROUND_TRUNC)) ? trunc(p) : rint(p);
  r = fmax(r, -(double)qmax);
  r = fmin(r, (double)qmax);
  return (int32_t)r;
}

static int32_t clamp_code(int32_t n, int qmax) {
  return n < -qmax ? -qmax : (n > qmax ? qmax : n);
}

/* Steps 6-8 for one row.  x: updated row; d: the row as stored before this
 * step, dequantized without decay (the BDR reference: a code's move is from
 * its stored value before the step to its stored value after it); Sp:
 * decayed row before the write (used only by the planted BDR_REFERENCE
 * mistake); R: updated shadow row or NULL. */
static void requantize_row(const qo_cfg* c, const float* x, const float* Sp,
                           const float* d, const float* R, const float* sigma,
                           int32_t* crow, float* srow, double* pre) {
  const int G = c->group, ng = c->dk / c->group, qmax = c->qmax;
  for (int g = 0; g < ng; ++g) {
    float s_new;
    int policy = c->policy;
    if (FAULT(QO_FAULT_PERSIST_UPDATE) && policy == QO_SCALE_PERSISTENT)
      policy = QO_SCALE_DYNAMIC;
    if (FAULT(QO_FAULT_YOKED_FROM_X) && policy == QO_SCALE_YOKED)
      policy = QO_SCALE_DYNAMIC;
    if (policy == QO_SCALE_PERSISTENT) {
      s_new = srow[g];
    } else {
      const float* src = (policy == QO_SCALE_YOKED) ? R : x;
      float m = 0.0f;
      for (int j = g * G; j < (g + 1) * G; ++j) m = fmaxf(m, fabsf(src[j]));
      s_new = m / (float)qmax;
    }
    if (!(s_new > 0.0f)) {
      for (int j = g * G; j < (g + 1) * G; ++j) {
        crow[j] = 0;
        if (pre) pre[j] = NAN;
      }
    } else {
      float inv = 1.0f / s_new;
      for (int j = g * G; j < (g + 1) * G; ++j) {
        int32_t n = nearest_code(x[j], inv, qmax, pre ? &pre[j] : NULL);
        if (c->rounding == QO_ROUND_BDR) {
          float ref = (FAULT(QO_FAULT_BDR_REFERENCE)) ? Sp[j] : d[j];
          float dq = (float)n * s_new;
          if (sigma[j] > 0.0f && dq < ref)
            n += 1;
          else if (sigma[j] < 0.0f && dq > ref)
            n -= 1;
          n = clamp_code(n, qmax);
        }
        crow[j] = n;
      }
    }
    srow[g] = s_new;
  }
}

int qo_init(const qo_cfg* c, const float* S0, int32_t* codes, float* scales,
            float* shadow) {
  if (qo_check(c) || !S0 || !codes || !scales) return -1;
  if (c->policy == QO_SCALE_YOKED && !shadow) return -1;
  const int dk = c->dk, dv = c->dv, G = c->group, ng = dk / G, qmax = c->qmax;
#pragma omp parallel for schedule(static)
  for (int t = 0; t < c->tiles; ++t) {
    for (int i = 0; i < dv; ++i) {
      size_t row = (size_t)t * dv + i;
      const float* x = S0 + row * dk;
      int32_t* crow = codes + row * dk;
      float* srow = scales + row * ng;
      for (int g = 0; g < ng; ++g) {
        float m = 0.0f;
        for (int j = g * G; j < (g + 1) * G; ++j) m = fmaxf(m, fabsf(x[j]));
        float s = m / (float)qmax;
        if (!(s > 0.0f)) {
          for (int j = g * G; j < (g + 1) * G; ++j) crow[j] = 0;
        } else {
          float inv = 1.0f / s;
          for (int j = g * G; j < (g + 1) * G; ++j)
            crow[j] = nearest_code(x[j], inv, qmax, NULL);
        }
        srow[g] = s;
      }
      if (shadow) memcpy(shadow + row * dk, x, sizeof(float) * dk);
    }
  }
  return 0;
}

int qo_step(const qo_cfg* c, int32_t* codes, float* scales, float* shadow,
            const float* q, const float* k, const float* v, const float* alpha,
            const float* beta, float* o, double* prequant) {
  if (qo_check(c) || !codes || !scales || !k || !v || !alpha || !beta) return -1;
  if (o && !q) return -1;
  if (c->policy == QO_SCALE_YOKED && !shadow) return -1;
  const int dk = c->dk, dv = c->dv, G = c->group, ng = dk / G;
#pragma omp parallel for schedule(static)
  for (int t = 0; t < c->tiles; ++t) {
    float d[QO_MAX_DK], Sp[QO_MAX_DK], x[QO_MAX_DK], Rp[QO_MAX_DK], Rn[QO_MAX_DK];
    float sg[QO_MAX_DK];
    const float* kt = k + (size_t)t * dk;
    const float* qt = q ? q + (size_t)t * dk : NULL;
    for (int i = 0; i < dv; ++i) {
      size_t row = (size_t)t * dv + i;
      int32_t* crow = codes + row * dk;
      float* srow = scales + row * ng;
      /* 1. dequantize with the decayed scale: S' = c * (s * a) */
      for (int j = 0; j < dk; ++j) {
        int g = j / G;
        if (FAULT(QO_FAULT_GROUP_INDEX)) g = (g + 1) % ng;
        d[j] = (float)crow[j] * srow[g];
        Sp[j] = (float)crow[j] * (srow[g] * decay_at(c, alpha, t, i, j));
      }
      /* 2-3. write */
      float w = row_write(c, Sp, kt, v[(size_t)t * dv + i], beta[t], x);
      /* 4. readout from the updated, not yet requantized row */
      if (o) o[row] = qo_dot(x, FAULT(QO_FAULT_READ_K_FOR_Q) ? kt : qt, dk);
      /* 5. yoked shadow */
      const float* R = NULL;
      if (c->policy == QO_SCALE_YOKED) {
        float* Rrow = shadow + row * dk;
        for (int j = 0; j < dk; ++j) Rp[j] = Rrow[j] * decay_at(c, alpha, t, i, j);
        row_write(c, Rp, kt, v[(size_t)t * dv + i], beta[t], Rn);
        memcpy(Rrow, Rn, sizeof(float) * dk);
        R = Rn;
      }
      /* 6-9. scale, round, store */
      for (int j = 0; j < dk; ++j) sg[j] = sign_of(w) * sign_of(kt[j]);
      requantize_row(c, x, Sp, d, R, sg, crow, srow, prequant ? prequant + row * dk : NULL);
    }
  }
  return 0;
}

int qo_lrb_step(const qo_cfg* c, int rank, int slot, int32_t* codes, float* scales,
                float* shadow, const float* A_in, float* A_out, const float* K_in,
                float* K_out, float* U, const float* q, const float* k, const float* v,
                const float* alpha, const float* beta, float* o, double* prequant) {
  if (qo_check(c) || rank < 1 || rank > QO_MAX_RANK || slot < 0 || slot >= rank) return -1;
  if (!codes || !scales || !k || !v || !alpha || !beta || !U) return -1;
  if (o && !q) return -1;
  if (c->policy == QO_SCALE_YOKED && !shadow) return -1;
  const int merge = slot == rank - 1;
  if (slot > 0 && (!A_in || !K_in)) return -1;
  if (!merge && (!A_out || !K_out)) return -1;
  const int dk = c->dk, dv = c->dv, G = c->group, ng = dk / G;
#pragma omp parallel for schedule(static)
  for (int t = 0; t < c->tiles; ++t) {
    float A[QO_MAX_DK], Kd[QO_MAX_RANK][QO_MAX_DK], kk[QO_MAX_RANK], kq[QO_MAX_RANK];
    float d[QO_MAX_DK], Sp[QO_MAX_DK], x[QO_MAX_DK], M[QO_MAX_DK], Rp[QO_MAX_DK], Rn[QO_MAX_DK];
    float sg[QO_MAX_DK];
    const float* kt = k + (size_t)t * dk;
    const float* qt = q ? q + (size_t)t * dk : NULL;
    float* Ut = U + (size_t)t * dv * rank;
    /* a. decay of the accumulated column factors and of the buffered keys */
    for (int j = 0; j < dk; ++j) {
      float a = decay_at(c, alpha, t, 0, j);
      A[j] = (slot == 0 ? 1.0f : A_in[(size_t)t * dk + j]) * a;
      for (int r = 0; r < slot; ++r) Kd[r][j] = K_in[((size_t)t * rank + r) * dk + j] * a;
    }
    /* b. the buffered keys against k and q */
    for (int r = 0; r < slot; ++r) {
      kk[r] = qo_dot(Kd[r], kt, dk);
      kq[r] = qt ? qo_dot(Kd[r], qt, dk) : 0.0f;
    }
    const float kqn = qt ? qo_dot(kt, qt, dk) : 0.0f;
    for (int i = 0; i < dv; ++i) {
      size_t row = (size_t)t * dv + i;
      int32_t* crow = codes + row * dk;
      float* srow = scales + row * ng;
      /* c. dequantize with the accumulated decay: S'_j = c * (s * A_j) */
      for (int j = 0; j < dk; ++j) {
        int g = j / G;
        if (FAULT(QO_FAULT_GROUP_INDEX)) g = (g + 1) % ng;
        d[j] = (float)crow[j] * srow[g];
        Sp[j] = (float)crow[j] * (srow[g] * A[j]);
      }
      /* d. write coefficient against the effective state S' + sum_r U_r K_r^T */
      float w;
      const float vi = v[row];
      if (c->delta && !FAULT(QO_FAULT_DROP_DELTA)) {
        float u = qo_dot(Sp, kt, dk);
        for (int r = 0; r < slot; ++r) u = fmaf(Ut[(size_t)i * rank + r], kk[r], u);
        w = (FAULT(QO_FAULT_BETA_ON_V_ONLY)) ? beta[t] * vi - u : beta[t] * (vi - u);
      } else {
        w = beta[t] * vi;
      }
      if (FAULT(QO_FAULT_WRITE_SIGN)) w = -w;
      /* yoked shadow: the FP32 reference advances every step */
      const float* R = NULL;
      if (c->policy == QO_SCALE_YOKED) {
        float* Rrow = shadow + row * dk;
        for (int j = 0; j < dk; ++j) Rp[j] = Rrow[j] * decay_at(c, alpha, t, i, j);
        row_write(c, Rp, kt, vi, beta[t], Rn);
        memcpy(Rrow, Rn, sizeof(float) * dk);
        R = Rn;
      }
      if (!merge) {
        /* e. bypass: the write joins the buffer; the stored state is untouched */
        if (o) {
          float oi = qo_dot(Sp, FAULT(QO_FAULT_READ_K_FOR_Q) ? kt : qt, dk);
          for (int r = 0; r < slot; ++r) oi = fmaf(Ut[(size_t)i * rank + r], kq[r], oi);
          o[row] = fmaf(w, kqn, oi);
        }
        Ut[(size_t)i * rank + slot] = w;
      } else {
        /* f. merge: x = S' + sum_r U_r K_r^T + w k^T, then requantize once */
        for (int j = 0; j < dk; ++j) {
          float xj = Sp[j], mj = 0.0f;
          for (int r = 0; r < slot; ++r) {
            const float ur = Ut[(size_t)i * rank + r];
            xj = fmaf(ur, Kd[r][j], xj);
            mj = fmaf(ur, Kd[r][j], mj);
          }
          x[j] = fmaf(w, kt[j], xj);
          M[j] = fmaf(w, kt[j], mj);
          sg[j] = FAULT(QO_FAULT_LRB_SIGN_LAST) ? sign_of(w) * sign_of(kt[j]) : sign_of(M[j]);
        }
        if (o) o[row] = qo_dot(x, FAULT(QO_FAULT_READ_K_FOR_Q) ? kt : qt, dk);
        requantize_row(c, x, Sp, d, R, sg, crow, srow, prequant ? prequant + row * dk : NULL);
      }
    }
    if (!merge) {
      memcpy(A_out + (size_t)t * dk, A, sizeof(float) * dk);
      for (int r = 0; r < slot; ++r)
        memcpy(K_out + ((size_t)t * rank + r) * dk, Kd[r], sizeof(float) * dk);
      memcpy(K_out + ((size_t)t * rank + slot) * dk, kt, sizeof(float) * dk);
    }
  }
  return 0;
}

int qo_readout(const qo_cfg* c, const int32_t* codes, const float* scales,
               const float* q, float* o) {
  if (qo_check(c) || !codes || !scales || !q || !o) return -1;
  const int dk = c->dk, dv = c->dv, G = c->group, ng = dk / G;
#pragma omp parallel for schedule(static)
  for (int t = 0; t < c->tiles; ++t) {
    float d[QO_MAX_DK];
    for (int i = 0; i < dv; ++i) {
      size_t row = (size_t)t * dv + i;
      for (int j = 0; j < dk; ++j) {
        int g = j / G;
        if (FAULT(QO_FAULT_GROUP_INDEX)) g = (g + 1) % ng;
        d[j] = (float)codes[row * dk + j] * scales[row * ng + g];
      }
      o[row] = qo_dot(d, q + (size_t)t * dk, dk);
    }
  }
  return 0;
}

int qo_sq_norms(const qo_cfg* c, const int32_t* codes, const float* scales, double* out) {
  if (qo_check(c) || !codes || !scales || !out) return -1;
  const int dk = c->dk, dv = c->dv, G = c->group, ng = dk / G;
#pragma omp parallel for schedule(static)
  for (int t = 0; t < c->tiles; ++t) {
    double acc = 0.0;
    for (int i = 0; i < dv; ++i) {
      size_t row = (size_t)t * dv + i;
      for (int j = 0; j < dk; ++j) {
        double d = (double)((float)codes[row * dk + j] * scales[row * ng + j / G]);
        acc += d * d;
      }
    }
    out[t] = acc;
  }
  return 0;
}

int qo_fp32_sq_norms(const qo_cfg* c, const float* S, double* out) {
  if (qo_check(c) || !S || !out) return -1;
  const size_t n = (size_t)c->dv * c->dk;
#pragma omp parallel for schedule(static)
  for (int t = 0; t < c->tiles; ++t) {
    double acc = 0.0;
    for (size_t e = 0; e < n; ++e) {
      double x = (double)S[(size_t)t * n + e];
      acc += x * x;
    }
    out[t] = acc;
  }
  return 0;
}

int qo_fp32_step(const qo_cfg* c, float* S, const float* q, const float* k,
                 const float* v, const float* alpha, const float* beta, float* o) {
  if (qo_check(c) || !S || !k || !v || !alpha || !beta) return -1;
  if (o && !q) return -1;
  const int dk = c->dk, dv = c->dv;
#pragma omp parallel for schedule(static)
  for (int t = 0; t < c->tiles; ++t) {
    float Sp[QO_MAX_DK], x[QO_MAX_DK];
    const float* kt = k + (size_t)t * dk;
    for (int i = 0; i < dv; ++i) {
      size_t row = (size_t)t * dv + i;
      float* Srow = S + row * dk;
      for (int j = 0; j < dk; ++j) Sp[j] = Srow[j] * decay_at(c, alpha, t, i, j);
      row_write(c, Sp, kt, v[row], beta[t], x);
      memcpy(Srow, x, sizeof(float) * dk);
      if (o)
        o[row] = qo_dot(x, FAULT(QO_FAULT_READ_K_FOR_Q) ? kt : q + (size_t)t * dk, dk);
    }
  }
  return 0;
}

int qo_pack(int bits, int64_t n, const int32_t* codes, uint8_t* packed) {
  if (!codes || !packed || n < 0) return -1;
  if (bits == 8) {
    for (int64_t e = 0; e < n; ++e) packed[e] = (uint8_t)(codes[e] & 0xFF);
    return 0;
  }
  if (bits == 4) {
    if (n % 2) return -1;
    for (int64_t e = 0; e < n; e += 2)
      packed[e / 2] = (uint8_t)((codes[e] & 0xF) | ((codes[e + 1] & 0xF) << 4));
    return 0;
  }
  return -1;
}

int qo_unpack(int bits, int64_t n, const uint8_t* packed, int32_t* codes) {
  if (!codes || !packed || n < 0) return -1;
  if (bits == 8) {
    for (int64_t e = 0; e < n; ++e) codes[e] = (int32_t)(int8_t)packed[e];
    return 0;
  }
  if (bits == 4) {
    if (n % 2) return -1;
    for (int64_t e = 0; e < n; ++e) {
      int nib = (packed[e / 2] >> (4 * (e % 2))) & 0xF;
      codes[e] = nib >= 8 ? nib - 16 : nib;
    }
    return 0;
  }
  return -1;
}
