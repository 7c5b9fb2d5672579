// Chunkwise prefill on the fifth-generation tensor cores (qstate_prefill_tf32):
// the same recurrence and regrouping as prefill_kernel (qstate_prefill.cuh),
// with the four contractions of a chunk issued as tcgen05.mma in TF32 and
// accumulated in FP32 in tensor memory (LinQuant, Low-Precision Chunkwise
// Realization: local score, state read, intra-chunk output, state write;
// the state pass is an FP32 scale of the accumulator).
//
// One CTA per tile at a time, persistent over tiles; chunks of C = 64
// tokens; 16 warps, four per quadrant of tensor-memory lanes (each takes a
// quarter of the columns).  Each thread holds the next chunk's inputs in
// registers: their loads are issued once the current chunk's output
// contraction is issued and land while it, the state write and the
// epilogues run.  Tensor memory (256 columns per CTA):
//   S   columns [0, Dk)     the FP32 state, row i of Dv in the lane of an
//                           M = MDV accumulator, held pre-scaled (below);
//                           it stays there for the whole sequence and is the
//                           A operand of the state read
//   X   columns [128, 192)  local scores D[t][s] (M = 64), then the output
//                           O^T[i][t] (M = MDV)
//   VT  columns [192, 256)  beta_s v^T[i][s] (A operand of the intra-chunk
//                           output and of the state write)
// Shared memory holds the smem operands unswizzled, element (r, k) of an
// R x K K-major operand at byte (r/8)*32K + (k/4)*128 + (r%8)*16 + (k%4)*4.
//
// Per chunk, with Lam the running log-decay (inclusive; per channel under
// diagonal decay), m the chunk's middle token and C its last:
//   Qs = q e^{Lam_t - Lam_m},  Ks = k e^{Lam_m - Lam_s}
//   S is held as P = S_in e^{Lam_m} (column j scaled by e^{Lam_mj})
//   scores  D[t][s] = sum_j Qs[t][j] Ks[s][j] = q_t . k_s e^{Lam_t - Lam_s}
//                                                     (M=64, N=64, K=Dk)
//   output  O^T = P Qs^T + VT A^T,  A = D masked to s <= t   (M=Dv, N=64)
//           (= S_in q_t e^{Lam_t} + sum_{s<=t} D[t][s] beta_s v_s)
//   state   P += VT KbT^T with KbT[j][s] = Ks[s][j], an exact transposed copy
//           formed while the scores run (M=Dv, N=Dk, K=64); then
//           S_out = P e^{Lam_C - Lam_m}, folded into the next chunk's
//           pre-scale (one FP32 pass over S per chunk) or into the store of
//           the tile's final state.
// The factors e^{+-(Lam_t - Lam_m)} stay in range while a chunk decays a
// channel by at most e^-170.
//
// Operands are rounded to TF32 (round to nearest, ties away) before they
// are stored; the state operand of the state read is the FP32 accumulator,
// which the tensor core reads at TF32 precision (low mantissa bits
// dropped).  Every mbarrier wait is bounded: on a timeout the kernel counts
// it in `timeouts`, frees its tensor memory and returns.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "qstate_prefill.cuh"

namespace qs {

constexpr int kTcChunk = 64;
constexpr int kTcThreads = 512;
constexpr int kTcCols = 256;
constexpr int kTcColS = 0, kTcColX = 128, kTcColV = 192;
// Shared memory per CTA is at least this, so that at most two CTAs (two
// 256-column tensor-memory allocations) share an SM.
constexpr int kTcMinSmem = 80 * 1024;
// mbarrier polls before a wait gives up (each poll may suspend the thread
// for a bounded, system-dependent time).
constexpr long long kTcSpinLimit = 1ll << 22;

struct TcLayout {
  int qs, ks, kbt, a, lam, beta, lamc, part, misc, total;
  __host__ __device__ TcLayout(int dk, bool diag) {
    constexpr int C = kTcChunk;
    int off = 0;
    qs = off;   off += C * dk * 4;   // A operand of the scores, B operand of the state read
    ks = off;   off += C * dk * 4;   // Ks: B operand of the scores
    kbt = off;  off += dk * C * 4;   // KbT[j][s] = Ks[s][j]: B operand of the state write
    a = off;    off += C * C * 4;    // local scores A[t][s], B operand of the intra-chunk output
    // diagonal: Lam[t][j] (row stride dk + 4); scalar: Lam[t], e^{Lam_t - Lam_m}, e^{Lam_m - Lam_t}
    lam = off;  off += diag ? C * (dk + 4) * 4 : 3 * C * 4;
    beta = off; off += C * 4;
    // per channel (diagonal) or one value (scalar): e^{Lam_m}, e^{Lam_C - Lam_m} of this
    // chunk and e^{Lam_C - Lam_m} of the previous chunk
    lamc = off; off += diag ? 3 * dk * 4 : 16;
    part = off; off += diag ? kTcThreads * 4 : 0;  // diagonal: per-thread partial log sums
    misc = off; off += 16;                         // mbarrier, tensor-memory base, failure flag
    total = off;
  }
  __host__ __device__ int bytes() const { return total > kTcMinSmem ? total : kTcMinSmem; }
};

namespace tc {

__device__ __forceinline__ uint32_t saddr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// byte offset of element (r, k) of a K-major operand with K columns
__device__ __forceinline__ uint32_t cm_off(int r, int k, int K) {
  return static_cast<uint32_t>((r >> 3) * (K * 32) + (k >> 2) * 128 + (r & 7) * 16 + (k & 3) * 4);
}

// Shared-memory matrix descriptor, K-major without swizzle: start address,
// 128 bytes between the two core matrices of one MMA's K step (leading
// byte offset), sbo bytes between 8-row groups (stride byte offset),
// descriptor version 1.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t sbo) {
  uint64_t d = static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(128u >> 4) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  return d;
}

// Instruction descriptor: FP32 accumulator, TF32 A and B, both K-major.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t mbar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
               : "memory");
}
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint32_t mbar) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mbar) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Wait for the phase with the given parity to complete; false after
// `limit` polls.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity, long long limit = kTcSpinLimit) {
  for (long long i = 0; i < limit; ++i) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(mbar), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

__device__ __forceinline__ float tf32(float x) {
  uint32_t y;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(y) : "f"(x));
  return __uint_as_float(y);
}

// 16 consecutive columns of this warp's 32 lanes (one register per column).
__device__ __forceinline__ void tm_ld16(uint32_t addr, float (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=f"(r[0]), "=f"(r[1]), "=f"(r[2]), "=f"(r[3]), "=f"(r[4]), "=f"(r[5]), "=f"(r[6]),
        "=f"(r[7]), "=f"(r[8]), "=f"(r[9]), "=f"(r[10]), "=f"(r[11]), "=f"(r[12]), "=f"(r[13]),
        "=f"(r[14]), "=f"(r[15])
      : "r"(addr));
}
__device__ __forceinline__ void tm_st16(uint32_t addr, const float (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(addr),
      "f"(r[0]), "f"(r[1]), "f"(r[2]), "f"(r[3]), "f"(r[4]), "f"(r[5]), "f"(r[6]), "f"(r[7]),
      "f"(r[8]), "f"(r[9]), "f"(r[10]), "f"(r[11]), "f"(r[12]), "f"(r[13]), "f"(r[14]), "f"(r[15])
      : "memory");
}

__device__ __forceinline__ void st_shared4(unsigned char* base, uint32_t off, float a, float b, float c,
                                           float d) {
  *reinterpret_cast<float4*>(base + off) = make_float4(a, b, c, d);
}

}  // namespace tc

// Row of an M-row accumulator held by lane `lane` of a warp of quadrant
// qd (warp % 4): M = 128 puts row r in lane r; M = 64 puts rows
// 16 qd .. 16 qd + 15 in lanes 32 qd .. 32 qd + 15.
template <int M>
__device__ __forceinline__ int tc_row(int qd, int lane) {
  return M == 128 ? 32 * qd + lane : (lane < 16 ? 16 * qd + lane : -1);
}

// One chunk's inputs held in registers by one thread: its Qs/Ks items (8
// tokens x 16 columns per warp step, a float4 of q and of k per lane), a
// quarter of its row of v^T, the scalar decays of two tokens and beta of
// one (diagonal decays are loaded when the chunk's scan runs).
template <int DK>
struct TcInputs {
  static constexpr int IQ = DK / 32;
  static constexpr int TP = kTcChunk * DK / kTcThreads;  // tokens per thread of the diagonal scan
  float4 q[IQ], k[IQ];
  float v[kTcChunk / 4];
  float a0, a1, b;
};

template <int DK>
__device__ __forceinline__ void tc_load(TcInputs<DK>& in, const PrefillParams& p, size_t tok0, int Ce,
                                        int warp, int lane, int irow, bool ivalid, bool diag) {
  constexpr int C = kTcChunk;
  constexpr int TP = TcInputs<DK>::TP;
#pragma unroll
  for (int i = 0; i < TcInputs<DK>::IQ; ++i) {
    const int it = warp + 16 * i;
    const int t = 8 * (it & 7) + (lane & 7);
    const int j = 16 * (it >> 3) + 4 * (lane >> 3);
    in.q[i] = in.k[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (t < Ce) {
      in.q[i] = __ldg(reinterpret_cast<const float4*>(p.q + (tok0 + t) * DK + j));
      in.k[i] = __ldg(reinterpret_cast<const float4*>(p.k + (tok0 + t) * DK + j));
    }
  }
  const int s0 = (C / 4) * (warp >> 2);
#pragma unroll
  for (int u = 0; u < C / 4; ++u)
    in.v[u] = (ivalid && s0 + u < Ce) ? __ldg(p.v + (tok0 + s0 + u) * p.dv + irow) : 0.0f;
  const int tid = 32 * warp + lane;
  in.a0 = in.a1 = 1.0f;
  if (!diag && warp == 0) {
    if (lane < Ce) in.a0 = __ldg(p.alpha + tok0 + lane);
    if (32 + lane < Ce) in.a1 = __ldg(p.alpha + tok0 + 32 + lane);
  }
  in.b = tid < Ce ? __ldg(p.beta + tok0 + tid) : 0.0f;
}

template <int DK, int MDV, bool DIAG>
__global__ void __launch_bounds__(kTcThreads, 1)
    prefill_tc_kernel(PrefillParams p, int tiles, unsigned int* timeouts) {
  using namespace tc;
  constexpr int C = kTcChunk;
  constexpr int LS = DK + 4;  // row stride of the diagonal-decay Lam table
  constexpr int NF = DIAG ? DK : 1;  // decay factors per chunk
  static_assert(DK == 64 || DK == 128, "Dk");
  static_assert(MDV == 64 || MDV == 128, "accumulator rows");
  static_assert(kTcThreads == 512, "16 warps: four per tensor-memory lane quadrant");
  extern __shared__ __align__(1024) unsigned char tsm[];
  const TcLayout Ly(DK, DIAG);
  unsigned char* sQs = tsm + Ly.qs;
  unsigned char* sKs = tsm + Ly.ks;
  unsigned char* sKbT = tsm + Ly.kbt;
  unsigned char* sA = tsm + Ly.a;
  float* lam = reinterpret_cast<float*>(tsm + Ly.lam);
  float* fq = lam + C;      // scalar: e^{Lam_t - Lam_m}
  float* fk = lam + 2 * C;  // scalar: e^{Lam_m - Lam_t}
  float* bt = reinterpret_cast<float*>(tsm + Ly.beta);
  float* pre = reinterpret_cast<float*>(tsm + Ly.lamc);  // e^{Lam_m}
  float* post = pre + NF;                                 // e^{Lam_C - Lam_m}
  float* carry = pre + 2 * NF;                            // the previous chunk's post
  uint64_t* mbar_p = reinterpret_cast<uint64_t*>(tsm + Ly.misc);
  volatile uint32_t* tslot = reinterpret_cast<volatile uint32_t*>(tsm + Ly.misc + 8);
  volatile int* failed = reinterpret_cast<volatile int*>(tsm + Ly.misc + 12);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3;   // tensor-memory lane quadrant of this warp
  const int qt = warp >> 2;  // which quarter of the columns this warp takes
  const int dv = p.dv;
  const uint32_t mbar = saddr(mbar_p);

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     saddr(const_cast<uint32_t*>(tslot))),
                 "r"(kTcCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    mbar_init(mbar);
    *failed = 0;
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tbase = *tslot;
  const uint32_t tw = tbase + (static_cast<uint32_t>(32 * qd) << 16);  // this warp's lanes
  uint32_t phase = 0;
  const int irow = tc_row<MDV>(qd, lane);  // state / output row of this lane
  const bool ivalid = irow >= 0 && irow < dv;
  const int trow = tc_row<64>(qd, lane);   // score row of this lane
  const int nch = (p.L + C - 1) / C;
  const int cS0 = qt * (DK / 4), cS1 = cS0 + DK / 4;  // this warp's state columns

  // Wait for the MMAs committed last: warp 0 polls, the barrier releases the
  // others.  On a timeout every thread leaves.
  auto wait_mma = [&]() -> bool {
    if (warp == 0 && !mbar_wait(mbar, phase)) *failed = 1;
    phase ^= 1u;
    __syncthreads();
    fence_after();
    return *failed == 0;
  };

  // Bounded-wait self-check: nothing has been committed, so this wait cannot
  // complete; it must give up after p.wait_probe polls, and the CTA then
  // skips all work, frees its tensor memory and returns.
  int ntiles = tiles;
  if (p.wait_probe > 0) {
    if (warp == 0 && !mbar_wait(mbar, phase, p.wait_probe)) *failed = 1;
    __syncthreads();
    ntiles = 0;
  }

  int tile = blockIdx.x, ch = 0;
  bool pending = false;   // the state write of the previous chunk is in flight
  TcInputs<DK> in;
  if (tile < ntiles) tc_load<DK>(in, p, static_cast<size_t>(tile) * p.L, min(C, p.L), warp, lane, irow, ivalid, DIAG);

  while (tile < ntiles) {
    const int c0 = ch * C;
    const int Ce = min(C, p.L - c0);
    const size_t tok0 = static_cast<size_t>(tile) * p.L + c0;
    const int m = (Ce - 1) / 2;

    // the previous chunk's readers of lam, beta and the factors are done
    __syncthreads();

    // ---- beta, the running log-decay and the decay factors (post moves to carry)
    if (tid < C) bt[tid] = in.b;
    if constexpr (DIAG) {
      // thread (j, part) scans TP tokens of channel j; the parts' totals are
      // then added in order
      constexpr int TP = C * DK / kTcThreads;
      float* psum = reinterpret_cast<float*>(tsm + Ly.part);
      const int j = tid % DK, pt = tid / DK;
      float acc = 0.0f, loc[TP];
#pragma unroll
      for (int u = 0; u < TP; ++u) {
        const int t = pt * TP + u;
        loc[u] = t < Ce ? __ldg(p.alpha + (tok0 + t) * DK + j) : 1.0f;
      }
#pragma unroll
      for (int u = 0; u < TP; ++u) {
        acc += logf(loc[u]);
        loc[u] = acc;
      }
      psum[pt * DK + j] = acc;
      __syncthreads();
      float off = 0.0f;
      for (int q2 = 0; q2 < pt; ++q2) off += psum[q2 * DK + j];
#pragma unroll
      for (int u = 0; u < TP; ++u) lam[(pt * TP + u) * LS + j] = loc[u] + off;
      __syncthreads();
      if (tid < DK) {
        const float lC = lam[(C - 1) * LS + tid], lm = lam[m * LS + tid];
        carry[tid] = ch == 0 ? 1.0f : post[tid];
        pre[tid] = expf(lm);
        post[tid] = expf(lC - lm);
      }
    } else {
      if (warp == 0) {
        float x0 = logf(in.a0), x1 = logf(in.a1);
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const float y0 = __shfl_up_sync(0xffffffffu, x0, d);
          const float y1 = __shfl_up_sync(0xffffffffu, x1, d);
          if (lane >= d) { x0 += y0; x1 += y1; }
        }
        x1 += __shfl_sync(0xffffffffu, x0, 31);
        const float lC = __shfl_sync(0xffffffffu, x1, 31);
        const float lm = __shfl_sync(0xffffffffu, m < 32 ? x0 : x1, m & 31);
        lam[lane] = x0;
        lam[32 + lane] = x1;
        fq[lane] = expf(x0 - lm);
        fq[32 + lane] = expf(x1 - lm);
        fk[lane] = expf(lm - x0);
        fk[32 + lane] = expf(lm - x1);
        if (lane == 0) {
          carry[0] = ch == 0 ? 1.0f : post[0];
          pre[0] = expf(lm);
          post[0] = expf(lC - lm);
        }
      }
    }
    __syncthreads();

    // ---- operands Qs, Ks from the registers (the previous chunk's state
    // write reads KbT and VT only)
#pragma unroll
    for (int i = 0; i < TcInputs<DK>::IQ; ++i) {
      const int itm = warp + 16 * i;
      const int t = 8 * (itm & 7) + (lane & 7);
      const int j = 16 * (itm >> 3) + 4 * (lane >> 3);
      const float4 qv = in.q[i], kv = in.k[i];
      const uint32_t o = cm_off(t, j, DK);
      if constexpr (DIAG) {
        const float4 lt = *reinterpret_cast<const float4*>(lam + t * LS + j);
        const float4 lm = *reinterpret_cast<const float4*>(lam + m * LS + j);
        st_shared4(sQs, o, tf32(qv.x * expf(lt.x - lm.x)), tf32(qv.y * expf(lt.y - lm.y)),
                   tf32(qv.z * expf(lt.z - lm.z)), tf32(qv.w * expf(lt.w - lm.w)));
        st_shared4(sKs, o, tf32(kv.x * expf(lm.x - lt.x)), tf32(kv.y * expf(lm.y - lt.y)),
                   tf32(kv.z * expf(lm.z - lt.z)), tf32(kv.w * expf(lm.w - lt.w)));
      } else {
        const float eq = fq[t], ek = fk[t];
        st_shared4(sQs, o, tf32(qv.x * eq), tf32(qv.y * eq), tf32(qv.z * eq), tf32(qv.w * eq));
        st_shared4(sKs, o, tf32(kv.x * ek), tf32(kv.y * ek), tf32(kv.z * ek), tf32(kv.w * ek));
      }
    }

    // ---- the previous chunk's state write has read VT and KbT and written S
    if (pending) {
      if (!wait_mma()) break;
      pending = false;
    }
    // ---- the initial state of a tile into tensor memory
    if (ch == 0) {
      const float* src = p.S + (static_cast<size_t>(tile) * dv + (ivalid ? irow : 0)) * DK;
#pragma unroll
      for (int c = cS0; c < cS1; c += 16) {
        float r[16];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float4 x = ivalid ? __ldg(reinterpret_cast<const float4*>(src + c) + u)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
          r[4 * u] = x.x; r[4 * u + 1] = x.y; r[4 * u + 2] = x.z; r[4 * u + 3] = x.w;
        }
        tm_st16(tw + kTcColS + c, r);
      }
      wait_st();
    }
    // ---- state pass: P <- P e^{Lam_C - Lam_m} (previous chunk) e^{Lam_m} (this chunk)
#pragma unroll
    for (int c = cS0; c < cS1; c += 16) {
      float r[16];
      tm_ld16(tw + kTcColS + c, r);
      wait_ld();
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int f = DIAG ? c + u : 0;
        r[u] *= carry[f] * pre[f];
      }
      tm_st16(tw + kTcColS + c, r);
    }
    // ---- VT[i][s] = beta_s v_si into tensor memory (this warp's rows, a quarter of the tokens)
    {
      float r[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) r[e] = tf32(bt[(C / 4) * qt + e] * in.v[e]);
      tm_st16(tw + kTcColV + (C / 4) * qt, r);
    }
    fence_async_smem();
    wait_st();
    fence_before();
    __syncthreads();  // Qs, Ks, VT, S complete

    // ---- local scores
    if (tid == 0) {
      fence_after();
      constexpr uint32_t id = idesc_tf32(64, C);
#pragma unroll
      for (int kk = 0; kk < DK / 8; ++kk)
        mma_ss(tbase + kTcColX, sdesc(saddr(sQs) + 256 * kk, DK * 32), sdesc(saddr(sKs) + 256 * kk, DK * 32),
               id, kk > 0);
      mma_commit(mbar);
    }
    // ---- while the scores run: KbT[j][s] = Ks[s][j] (an exact copy)
#pragma unroll
    for (int i = 0; i < DK / 32; ++i) {
      const int itm = warp + 16 * i;
      const int j = 8 * (itm % (DK / 8)) + (lane & 7);
      const int s = 16 * (itm / (DK / 8)) + 4 * (lane >> 3);
      float w[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) w[u] = *reinterpret_cast<const float*>(sKs + cm_off(s + u, j, DK));
      st_shared4(sKbT, cm_off(j, s, C), w[0], w[1], w[2], w[3]);
    }
    fence_async_smem();
    if (!wait_mma()) break;

    // ---- A[t][s] = D[t][s] for s <= t
#pragma unroll
    for (int s0 = (C / 4) * qt; s0 < (C / 4) * (qt + 1); s0 += 16) {
      float r[16];
      tm_ld16(tw + kTcColX + s0, r);
      wait_ld();
      if (trow >= 0) {
        const int t = trow;
#pragma unroll
        for (int u = 0; u < 16; u += 4) {
          float a[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) a[e] = (s0 + u + e <= t && t < Ce) ? tf32(r[u + e]) : 0.0f;
          st_shared4(sA, cm_off(t, s0 + u, C), a[0], a[1], a[2], a[3]);
        }
      }
    }
    fence_async_smem();
    fence_before();
    __syncthreads();

    // ---- outputs: state read + intra-chunk output, O^T in X
    if (tid == 0) {
      fence_after();
      constexpr uint32_t id = idesc_tf32(MDV, C);
#pragma unroll
      for (int kk = 0; kk < DK / 8; ++kk)
        mma_ts(tbase + kTcColX, tbase + kTcColS + 8 * kk, sdesc(saddr(sQs) + 256 * kk, DK * 32), id, kk > 0);
#pragma unroll
      for (int kk = 0; kk < C / 8; ++kk)
        mma_ts(tbase + kTcColX, tbase + kTcColV + 8 * kk, sdesc(saddr(sA) + 256 * kk, C * 32), id, 1u);
      mma_commit(mbar);
    }
    // ---- the next chunk's loads, in flight from here to the next chunk's staging
    int ntile = tile, nchk = ch + 1;
    if (nchk == nch) { nchk = 0; ntile += gridDim.x; }
    if (ntile < ntiles)
      tc_load<DK>(in, p, static_cast<size_t>(ntile) * p.L + nchk * C, min(C, p.L - nchk * C), warp, lane,
                  irow, ivalid, DIAG);
    if (!wait_mma()) break;

    // ---- state write: P += VT Ks^T, in flight while the outputs are written
    if (tid == 0) {
      fence_after();
      constexpr uint32_t id = idesc_tf32(MDV, DK);
#pragma unroll
      for (int kk = 0; kk < C / 8; ++kk)
        mma_ts(tbase + kTcColS, tbase + kTcColV + 8 * kk, sdesc(saddr(sKbT) + 256 * kk, C * 32), id, 1u);
      mma_commit(mbar);
    }
    pending = true;
    if (p.o != nullptr) {
#pragma unroll
      for (int t0 = (C / 4) * qt; t0 < (C / 4) * (qt + 1); t0 += 16) {
        float r[16];
        tm_ld16(tw + kTcColX + t0, r);
        wait_ld();
        if (ivalid) {
#pragma unroll
          for (int u = 0; u < 16; ++u)
            if (t0 + u < Ce) p.o[(tok0 + t0 + u) * dv + irow] = r[u];
        }
      }
    }
    fence_before();

    // ---- final state of the tile: S_out = P e^{Lam_C - Lam_m}
    if (ch == nch - 1) {
      if (!wait_mma()) break;
      pending = false;
      float* dst = p.S + (static_cast<size_t>(tile) * dv + (ivalid ? irow : 0)) * DK;
#pragma unroll
      for (int c = cS0; c < cS1; c += 16) {
        float r[16];
        tm_ld16(tw + kTcColS + c, r);
        wait_ld();
        if (ivalid) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int f = DIAG ? c + 4 * u : 0;
            reinterpret_cast<float4*>(dst + c)[u] =
                make_float4(r[4 * u] * post[f], r[4 * u + 1] * post[DIAG ? f + 1 : 0],
                            r[4 * u + 2] * post[DIAG ? f + 2 : 0], r[4 * u + 3] * post[DIAG ? f + 3 : 0]);
          }
        }
      }
      fence_before();
    }
    tile = ntile;
    ch = nchk;
  }

  __syncthreads();
  if (tid == 0 && *failed) atomicAdd(timeouts, 1u);
  fence_after();
  // On the timeout path a committed tcgen05.mma may still be writing these
  // tensor-memory columns when they are freed here (that is what the wait
  // gave up on), so the launch's S and o are undefined once a timeout is
  // counted; the caller checks the count.
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(kTcCols) : "memory");
}

}  // namespace qs
