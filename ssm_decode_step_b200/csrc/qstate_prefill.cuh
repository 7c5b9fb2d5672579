// Chunkwise prefill on an FP32 state: qstate_prefill.  The state S_0 that
// the quantized decode path then starts from (LinQuant, Low-Precision
// Chunkwise Realization, for the Mamba-2 family: state write, state pass,
// state read, local score, intra-chunk output; here in FP32, with the
// diagonal decay of the GLA family as the per-channel extension, and the
// delta-rule write of the DeltaNet family, LinQuant's "delta-rule updates").
//
// Per tile, tokens are taken in chunks of C = 32.  With Lam_t the running
// sum of log(alpha) over the chunk's tokens up to t (per channel for
// diagonal decay) and S the state at the chunk's start:
//   o_t   = (S (q_t * e^{Lam_t})) + sum_{s <= t} A_ts beta_s v_s
//   A_ts  = sum_j q_tj k_sj e^{Lam_tj - Lam_sj}
//   S_new = S * e^{Lam_C} + sum_s beta_s v_s (k_s * e^{Lam_C - Lam_s})^T
// which is the token-by-token recurrence S_t = S_{t-1} Lambda_t + beta_t v_t
// k_t^T, o_t = S_t q_t regrouped (exactly in real arithmetic).  Under scalar
// decay A_ts = (q_t . k_s) e^{Lam_t - Lam_s}; under diagonal decay the
// factor is split around the chunk's middle token m as
// (q_t e^{Lam_t - Lam_m}) . (k_s e^{Lam_m - Lam_s}), which stays in range
// while a chunk decays any channel by less than e^{-170}.
//
// Delta rule (delta = 1).  The recurrence
// S_t = S_{t-1} Lambda_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T is the
// linear write S_t = S_{t-1} Lambda_t + w_t k_t^T with the corrected value
//   w_t = beta_t (v_t - S_{t-1} Lambda_t k_t),
// and unrolling S_{t-1} over the chunk gives
//   w_t = beta_t (v_t - S (k_t * e^{Lam_t})) - sum_{s < t} B_ts w_s,
//   B_ts = beta_t sum_j k_tj k_sj e^{Lam_tj - Lam_sj},
// a unit lower-triangular system, solved by forward substitution (tokens in
// order, s ascending); w then takes the place of beta_s v_s in the output
// and the state pass (A without beta).  B is split around the middle token
// like A.
//
// One CTA per tile, 256 threads; the state stays in shared memory (rows
// padded to Dk + 1 floats) for the whole sequence.  Only the state pass is
// sequential; tiles are independent.
#pragma once

#include <cstdint>
#include <type_traits>
#include <cuda_runtime.h>

namespace qs {

constexpr int kPrefillChunk = 32;
// Threads per CTA: 256 where two CTAs fit on an SM, 512 (one CTA) where the
// state and the chunk buffers take more than half of the shared memory.
constexpr int kPrefillThreads = 256;
constexpr int kPrefillThreadsWide = 512;

struct PrefillParams {
  float* S;            // [T][dv][dk], in: initial state, out: state after the L tokens
  const float* q;      // [T][L][dk]
  const float* k;      // [T][L][dk]
  const float* v;      // [T][L][dv]
  const float* alpha;  // [T][L] (scalar) or [T][L][dk] (diagonal)
  const float* beta;   // [T][L]
  float* o;            // [T][L][dv] or nullptr
  int L;
  int dv;
  int wait_probe;      // tensor-core path only: > 0 runs the bounded-wait self-check instead
};

// Row stride of V in shared memory: a multiple of 32 plus 8 floats.  Lanes
// on consecutive rows i read consecutive banks; in the delta rule's split
// substitution the 4 lanes of a row read tokens s = sub + 4k, whose rows
// then start 8 banks apart, so the 8 rows x 4 lanes of a warp hit 32
// different banks.
__host__ __device__ constexpr int prefill_vs(int dv) { return (dv + 31) / 32 * 32 + 8; }

// Shared-memory layout (floats) of one CTA.
struct PrefillLayout {
  int S, qbar, kg, kbar, qt, kh, kq, v, lam, A, B, beta, elam, total;
  __host__ __device__ PrefillLayout(int dk, int dv, bool diag, bool delta = false) {
    constexpr int C = kPrefillChunk;
    int off = 0;
    S = off;    off += dv * (dk + 1);
    qbar = off; off += dk * (C + 4);     // [j][t]: q_t * e^{Lam_t} (rows padded to C + 4)
    kg = off;   off += delta ? dk * (C + 4) : 0;  // delta rule: [j][t] k_t * e^{Lam_t}, same padding
    kbar = off; off += C * dk;           // [s][j]: k_s * e^{Lam_C - Lam_s}
    qt = off;   off += C * (dk + 4);     // [t][j]: q_t (* e^{Lam_t - Lam_m} when diagonal)
    kh = off;   off += C * (dk + 4);     // [s][j]: k_s (* e^{Lam_m - Lam_s} when diagonal)
    // delta rule, diagonal decay: [t][j] k_t * e^{Lam_t - Lam_m} (scalar decay uses kh)
    kq = off;   off += (delta && diag) ? C * (dk + 4) : 0;
    // [s][i]: v, then w (delta rule); row stride = 8 mod 32 floats (prefill_vs)
    v = off;    off += C * prefill_vs(dv);
    lam = off;  off += diag ? C * dk : C;  // [t][j] or [t]
    A = off;    off += C * C;            // [t][s], beta_s folded in (linear write only)
    B = off;    off += delta ? C * C : 0;  // [t][s], s < t: the delta rule's triangular system
    beta = off; off += C;
    elam = off; off += diag ? dk : 1;    // e^{Lam_C} per channel
    total = off;
  }
};

// State read of two rows for TT (4 or 8) tokens: a[u] = sum_j r0[j] x[j][u],
// b[u] = sum_j r1[j] x[j][u], j ascending (x rows xs floats apart, 16-byte
// aligned).
template <int DK, int TT>
__device__ __forceinline__ void state_read2(const float* r0, const float* r1, const float* x, int xs,
                                            float (&a)[TT], float (&b)[TT]) {
#pragma unroll
  for (int u = 0; u < TT; ++u) a[u] = b[u] = 0.0f;
  for (int j = 0; j < DK; ++j) {
    const float s0 = r0[j], s1 = r1[j];
#pragma unroll
    for (int h = 0; h < TT / 4; ++h) {
      const float4 xv = *reinterpret_cast<const float4*>(x + j * xs + 4 * h);
      a[4 * h + 0] = fmaf(s0, xv.x, a[4 * h + 0]); a[4 * h + 1] = fmaf(s0, xv.y, a[4 * h + 1]);
      a[4 * h + 2] = fmaf(s0, xv.z, a[4 * h + 2]); a[4 * h + 3] = fmaf(s0, xv.w, a[4 * h + 3]);
      b[4 * h + 0] = fmaf(s1, xv.x, b[4 * h + 0]); b[4 * h + 1] = fmaf(s1, xv.y, b[4 * h + 1]);
      b[4 * h + 2] = fmaf(s1, xv.z, b[4 * h + 2]); b[4 * h + 3] = fmaf(s1, xv.w, b[4 * h + 3]);
    }
  }
}

template <int DK, bool DIAG, bool DELTA, int NT>
__global__ void __launch_bounds__(NT, NT == kPrefillThreads ? 2 : 1) prefill_kernel(PrefillParams p) {
  constexpr int C = kPrefillChunk;
  constexpr int TPW = C * 32 / NT;  // tokens per warp in the local scores
  extern __shared__ __align__(16) float sm[];
  const int dv = p.dv;
  const PrefillLayout Ly(DK, dv, DIAG, DELTA);
  float* S = sm + Ly.S;
  float* qbar = sm + Ly.qbar;
  float* kg = sm + Ly.kg;
  float* kbar = sm + Ly.kbar;
  float* qt = sm + Ly.qt;
  float* kh = sm + Ly.kh;
  float* kq = DIAG ? sm + Ly.kq : kh;
  float* V = sm + Ly.v;
  float* lam = sm + Ly.lam;
  float* A = sm + Ly.A;
  float* Bm = sm + Ly.B;
  float* bt = sm + Ly.beta;
  float* elam = sm + Ly.elam;
  const int tid = threadIdx.x;
  const size_t tile = blockIdx.x;
  constexpr int SP = DK + 1;  // padded state row
  constexpr int QP = DK + 4;  // padded q / k row (16-byte aligned, no bank conflicts)
  const int hv = dv / 2;      // rows i and i + hv go to one thread (dv is a multiple of 16)
  const int VS = prefill_vs(dv);  // padded row of V
  constexpr int QB = C + 4;   // padded qbar row: float4 stores of 4 tokens by consecutive j
                              // land in 8 different bank groups
  static_assert((NT == 256 || NT == 512) && C == 32, "8 or 16 warps, 32 keys");

  float* Sg = p.S + tile * dv * DK;
  for (int e = tid; e < dv * DK; e += NT) S[(e / DK) * SP + (e % DK)] = Sg[e];

  for (int c0 = 0; c0 < p.L; c0 += C) {
    const int Ce = min(C, p.L - c0);
    const size_t tok0 = tile * p.L + c0;
    __syncthreads();
    // ---- chunk inputs
    for (int e = tid; e < C * dv; e += NT) {
      const int s = e / dv, i = e % dv;
      V[s * VS + i] = s < Ce ? p.v[(tok0 + s) * dv + i] : 0.0f;
    }
    if (tid < C) bt[tid] = tid < Ce ? p.beta[tok0 + tid] : 0.0f;
    // ---- running log-decay over the chunk
    if constexpr (DIAG) {
      for (int j = tid; j < DK; j += NT) {
        float acc = 0.0f;
        for (int t = 0; t < C; ++t) {
          if (t < Ce) acc += logf(p.alpha[(tok0 + t) * DK + j]);
          lam[t * DK + j] = acc;
        }
        elam[j] = expf(acc);
      }
    } else {
      if (tid < 32) {
        float x = tid < Ce ? logf(p.alpha[tok0 + tid]) : 0.0f;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const float y = __shfl_up_sync(0xffffffffu, x, d);
          if (tid >= d) x += y;
        }
        lam[tid] = x;
        const float total = __shfl_sync(0xffffffffu, x, 31);
        if (tid == 0) elam[0] = expf(total);
      }
    }
    __syncthreads();
    // ---- decayed copies of q and k
    const int m = (Ce - 1) / 2;
    // thread (j, 4 tokens): global reads coalesced along j, one float4 of qbar
    for (int e = tid; e < DK * (C / 4); e += NT) {
      const int j = e % DK, t0 = 4 * (e / DK);
      float xb[4], gb[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = t0 + u;
        const bool live = t < Ce;
        const float qv = live ? p.q[(tok0 + t) * DK + j] : 0.0f;
        const float kv = live ? p.k[(tok0 + t) * DK + j] : 0.0f;
        if constexpr (DIAG) {
          const float lt = lam[t * DK + j], lC = lam[(C - 1) * DK + j], lm = lam[m * DK + j];
          const float el = expf(lt);
          xb[u] = qv * el;
          gb[u] = kv * el;  // delta rule: the keys' projection on the state
          kbar[t * DK + j] = kv * expf(lC - lt);
          qt[t * QP + j] = qv * expf(lt - lm);
          kh[t * QP + j] = kv * expf(lm - lt);
          if constexpr (DELTA) kq[t * QP + j] = kv * expf(lt - lm);
        } else {
          const float lt = lam[t], lC = lam[C - 1];
          const float el = expf(lt);
          xb[u] = qv * el;
          gb[u] = kv * el;
          kbar[t * DK + j] = kv * expf(lC - lt);
          qt[t * QP + j] = qv;
          kh[t * QP + j] = kv;
        }
      }
      *reinterpret_cast<float4*>(qbar + j * QB + t0) = make_float4(xb[0], xb[1], xb[2], xb[3]);
      if constexpr (DELTA)
        *reinterpret_cast<float4*>(kg + j * QB + t0) = make_float4(gb[0], gb[1], gb[2], gb[3]);
    }
    __syncthreads();
    // ---- local scores A_ts (s <= t), beta_s folded in: warp w takes tokens
    // t = TPW w .. TPW w + TPW - 1, lane s one key; float4 steps along Dk
    {
      const int lane = tid & 31, w = tid >> 5;
      const int s = lane;
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      float bcc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      const float4* kr = reinterpret_cast<const float4*>(kh + s * QP);
      for (int j4 = 0; j4 < DK / 4; ++j4) {
        const float4 kv = kr[j4];
#pragma unroll
        for (int u = 0; u < TPW; ++u) {
          const float4 qv = reinterpret_cast<const float4*>(qt + (TPW * w + u) * QP)[j4];
          acc[u] = fmaf(qv.x, kv.x, acc[u]);
          acc[u] = fmaf(qv.y, kv.y, acc[u]);
          acc[u] = fmaf(qv.z, kv.z, acc[u]);
          acc[u] = fmaf(qv.w, kv.w, acc[u]);
          if constexpr (DELTA) {
            const float4 kt = reinterpret_cast<const float4*>(kq + (TPW * w + u) * QP)[j4];
            bcc[u] = fmaf(kt.x, kv.x, bcc[u]);
            bcc[u] = fmaf(kt.y, kv.y, bcc[u]);
            bcc[u] = fmaf(kt.z, kv.z, bcc[u]);
            bcc[u] = fmaf(kt.w, kv.w, bcc[u]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < TPW; ++u) {
        const int t = TPW * w + u;
        const float f = (!DIAG && s <= t && t < Ce) ? expf(lam[t] - lam[s]) : 1.0f;
        float a = 0.0f;
        if (s <= t && t < Ce) {
          a = acc[u] * f;
          if constexpr (!DELTA) a *= bt[s];
        }
        A[t * C + s] = a;
        if constexpr (DELTA) Bm[t * C + s] = (s < t && t < Ce) ? bt[t] * (bcc[u] * f) : 0.0f;
      }
    }
    __syncthreads();
    if constexpr (DELTA) {
      // ---- r_t = beta_t (v_t - S (k_t e^{Lam_t})), in place of v (rows i, i + dv/2;
      // TT tokens per thread)
      auto project = [&](auto tt) {
        constexpr int TT = decltype(tt)::value;
        for (int e = tid; e < hv * (C / TT); e += NT) {
          const int i0 = e % hv, i1 = i0 + hv, tg = e / hv;
          float a0[TT], a1[TT];
          state_read2<DK, TT>(S + i0 * SP, S + i1 * SP, kg + TT * tg, QB, a0, a1);
#pragma unroll
          for (int u = 0; u < TT; ++u) {
            const int t = TT * tg + u;
            V[t * VS + i0] = bt[t] * (V[t * VS + i0] - a0[u]);
            V[t * VS + i1] = bt[t] * (V[t * VS + i1] - a1[u]);
          }
        }
      };
      if (hv * (C / 8) >= NT) project(std::integral_constant<int, 8>{});
      else project(std::integral_constant<int, 4>{});
      __syncthreads();
      // ---- forward substitution: w_t = r_t - sum_{s < t} B_ts w_s, P lanes of one
      // warp per row (partial sums over s = sub, sub + P, ..., then added by shuffles;
      // V's row stride keeps the lanes of a warp on different banks)
      auto solve = [&](auto pp) {
        constexpr int PL = decltype(pp)::value;
        const int sub = tid % PL;
        for (int base = tid - sub; base < PL * dv; base += NT) {
          const int i = base / PL;
          for (int t = 1; t < Ce; ++t) {
            float part = 0.0f;
            for (int s2 = sub; s2 < t; s2 += PL) part = fmaf(Bm[t * C + s2], V[s2 * VS + i], part);
#pragma unroll
            for (int d = 1; d < PL; d <<= 1) part += __shfl_xor_sync(0xffffffffu, part, d);
            if (sub == 0) V[t * VS + i] -= part;
            __syncwarp();
          }
        }
      };
      // 2 dv and 4 dv are multiples of 32, so every warp is wholly inside or
      // outside the rows of each pass (the shuffles and __syncwarp need all lanes)
      if (NT >= 4 * dv) solve(std::integral_constant<int, 4>{});
      else solve(std::integral_constant<int, 2>{});
      __syncthreads();
    }
    // ---- outputs: state read + intra-chunk output
    if (p.o != nullptr) {
      auto outputs = [&](auto tt) {
        constexpr int TT = decltype(tt)::value;
        for (int e = tid; e < hv * (C / TT); e += NT) {
          const int i0 = e % hv, i1 = i0 + hv, tg = e / hv;  // rows i, i + dv/2; TT tokens
          float a0[TT], a1[TT];
          state_read2<DK, TT>(S + i0 * SP, S + i1 * SP, qbar + TT * tg, QB, a0, a1);
          for (int s = 0; s < C; ++s) {
            const float v0 = V[s * VS + i0], v1 = V[s * VS + i1];
#pragma unroll
            for (int u = 0; u < TT; ++u) {
              const float a = A[(TT * tg + u) * C + s];
              a0[u] = fmaf(a, v0, a0[u]);
              a1[u] = fmaf(a, v1, a1[u]);
            }
          }
#pragma unroll
          for (int u = 0; u < TT; ++u) {
            const int t = TT * tg + u;
            if (t < Ce) {
              p.o[(tok0 + t) * dv + i0] = a0[u];
              p.o[(tok0 + t) * dv + i1] = a1[u];
            }
          }
        }
      };
      if (hv * (C / 8) >= NT) outputs(std::integral_constant<int, 8>{});
      else outputs(std::integral_constant<int, 4>{});
      __syncthreads();
    }
    // ---- state pass: S = S e^{Lam_C} + sum_s beta_s v_s kbar_s^T
    {
      constexpr int JW = 16;  // columns per thread, rows i and i + dv/2
      for (int e = tid; e < hv * (DK / JW); e += NT) {
        const int i0 = e % hv, i1 = i0 + hv, jb = (e / hv) * JW;
        float a0[JW], a1[JW];
        float* s0 = S + i0 * SP + jb;
        float* s1 = S + i1 * SP + jb;
#pragma unroll
        for (int u = 0; u < JW; ++u) {
          const float f = elam[DIAG ? jb + u : 0];
          a0[u] = s0[u] * f;
          a1[u] = s1[u] * f;
        }
        for (int s = 0; s < Ce; ++s) {
          const float w0 = DELTA ? V[s * VS + i0] : bt[s] * V[s * VS + i0];
          const float w1 = DELTA ? V[s * VS + i1] : bt[s] * V[s * VS + i1];
          const float4* kr = reinterpret_cast<const float4*>(kbar + s * DK + jb);
#pragma unroll
          for (int u4 = 0; u4 < JW / 4; ++u4) {
            const float4 kv = kr[u4];
            a0[4 * u4 + 0] = fmaf(w0, kv.x, a0[4 * u4 + 0]);
            a0[4 * u4 + 1] = fmaf(w0, kv.y, a0[4 * u4 + 1]);
            a0[4 * u4 + 2] = fmaf(w0, kv.z, a0[4 * u4 + 2]);
            a0[4 * u4 + 3] = fmaf(w0, kv.w, a0[4 * u4 + 3]);
            a1[4 * u4 + 0] = fmaf(w1, kv.x, a1[4 * u4 + 0]);
            a1[4 * u4 + 1] = fmaf(w1, kv.y, a1[4 * u4 + 1]);
            a1[4 * u4 + 2] = fmaf(w1, kv.z, a1[4 * u4 + 2]);
            a1[4 * u4 + 3] = fmaf(w1, kv.w, a1[4 * u4 + 3]);
          }
        }
#pragma unroll
        for (int u = 0; u < JW; ++u) {
          s0[u] = a0[u];
          s1[u] = a1[u];
        }
      }
    }
  }
  __syncthreads();
  for (int e = tid; e < dv * DK; e += NT) Sg[e] = S[(e / DK) * SP + (e % DK)];
}

}  // namespace qs
