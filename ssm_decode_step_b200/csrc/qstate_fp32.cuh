// Decode step of the unquantized FP32 recurrence (the baseline the quantized
// state is compared against): the same definition as include/qstate.h
// without codes and scales, S_t = S_{t-1} Lambda (I - delta beta k k^T) +
// beta v k^T and o = S_t q, in the same fixed FP32 order.  Same structure as
// step_kernel: persistent 128-thread CTAs over row blocks, a cp.async ring
// per CTA, packed FP32 on adjacent-column pairs.
#pragma once

#include "qstate_kernels.cuh"

namespace qs {

struct Fp32Layout {
  int S, v, k, q, a, misc, bytes;
  __host__ __device__ Fp32Layout(int dk, int rb, bool diag) {
    const int vec = (dk / 32) * kChunkStride * 4;
    int off = 0;
    S = off;    off += rb * dk * 4;
    v = off;    off = align_up(off + rb * 4, 16);
    k = off;    off += vec;
    q = off;    off += vec;
    a = off;    off += diag ? vec : 0;
    misc = off; off += 16;
    bytes = align_up(off, 128);
  }
};

template <int DK, bool DIAG>
__device__ __forceinline__ void fp32_stage_load(unsigned char* st, const Fp32Layout& L,
                                                const StepParams& p, const UnitCursor& u) {
  constexpr int VU = DK / 4;
  const int tid = threadIdx.x;
  const int rb = p.rb;
  const size_t tile = static_cast<size_t>(u.tile);
  const size_t row0 = u.row0(p);
  {
    // 16-byte unit i of local row-chunk rc at unit position i ^ (rc & 7)
    const int n16 = rb * DK / 4;
    const float* g = p.shadow + row0 * DK;
    for (int i = tid; i < n16; i += kThreads) {
      const int rc = i >> 3, w = i & 7;
      cp_async16(st + L.S + rc * 128 + 16 * (w ^ (rc & 7)), g + 4 * i);
    }
  }
  for (int i = tid; i < 3 * VU; i += kThreads) {
    const int which = i / VU, w = i % VU;
    if (which == 0) {
      cp_async16(st + L.k + vec_unit_offset(w), p.k + tile * DK + 4 * w);
    } else if (which == 1) {
      if (p.o != nullptr) cp_async16(st + L.q + vec_unit_offset(w), p.q + tile * DK + 4 * w);
    } else {
      if (DIAG) cp_async16(st + L.a + vec_unit_offset(w), p.alpha + tile * DK + 4 * w);
    }
  }
  for (int i = tid; i < rb / 4; i += kThreads) cp_async16(st + L.v + 16 * i, p.v + row0 + 4 * i);
  if (tid == kThreads - 1) {
    float* misc = reinterpret_cast<float*>(st + L.misc);
    if constexpr (!DIAG) cp_async4(misc + 0, p.alpha + tile);
    cp_async4(misc + 1, p.beta + tile);
  }
}

// p.shadow carries the FP32 state S [T][Dv][Dk].
template <int DK, bool DELTA, bool DIAG, int STAGES>
__global__ void __launch_bounds__(kThreads, QS_MIN_BLOCKS) fp32_step_kernel(StepParams p) {
  constexpr int LPR = DK / 32;
  constexpr int RP = kThreads / LPR;
  extern __shared__ __align__(128) unsigned char smem[];
  const Fp32Layout L(DK, p.rb, DIAG);
  const int tid = threadIdx.x;
  const int c = tid % LPR, r0 = tid / LPR;
  const bool readout = p.o != nullptr;
  grid_dep_wait();
  grid_dep_launch();

  UnitCursor pre(blockIdx.x, p);
#pragma unroll
  for (int s = 0; s < STAGES - 1; ++s) {
    if (pre.tile < p.tiles) fp32_stage_load<DK, DIAG>(smem + s * L.bytes, L, p, pre);
    cp_async_commit();
    pre.advance(p);
  }
  int it = 0;
  for (UnitCursor cur(blockIdx.x, p); cur.tile < p.tiles; cur.advance(p), ++it) {
    if (pre.tile < p.tiles) fp32_stage_load<DK, DIAG>(smem + ((it + STAGES - 1) % STAGES) * L.bytes, L, p, pre);
    cp_async_commit();
    pre.advance(p);
    cp_async_wait<STAGES - 1>();
    __syncthreads();
    unsigned char* st = smem + (it % STAGES) * L.bytes;
    const size_t grow0 = cur.row0(p);
    float2 kk[16];
    load_pairs(st + L.k, c, kk);
    const float* miscf = reinterpret_cast<const float*>(st + L.misc);
    const float beta = miscf[1];
    const float a_scalar = DIAG ? 1.0f : miscf[0];
#pragma unroll 1
    for (int r = r0; r < p.rb; r += RP) {
      const int rc = r * LPR + c;
      const float4* rs = reinterpret_cast<const float4*>(st + L.S + rc * 128);
      float2 x[16];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float4 t = rs[u ^ (rc & 7)];
        x[2 * u] = make_float2(t.x, t.y);
        x[2 * u + 1] = make_float2(t.z, t.w);
      }
      // S' = S * a
      if constexpr (DIAG) {
        float2 aa[16];
        load_pairs(st + L.a, c, aa);
#pragma unroll
        for (int m = 0; m < 16; ++m) x[m] = __fmul2_rn(x[m], aa[m]);
      } else {
#pragma unroll
        for (int m = 0; m < 16; ++m) x[m] = __fmul2_rn(x[m], f2(a_scalar));
      }
      const float v_i = reinterpret_cast<const float*>(st + L.v)[r];
      float wcoef;
      if constexpr (DELTA) {
        wcoef = __fmul_rn(beta, __fsub_rn(v_i, row_tree<LPR>(chunk_sum(x, kk))));
      } else {
        wcoef = __fmul_rn(beta, v_i);
      }
#pragma unroll
      for (int m = 0; m < 16; ++m) x[m] = __ffma2_rn(f2(wcoef), kk[m], x[m]);
      if (readout) {
        float2 qv[16];
        load_pairs(st + L.q, c, qv);
        const float o = row_tree<LPR>(chunk_sum(x, qv));
        if (c == 0) p.o[grow0 + r] = o;
      }
      float* dst = p.shadow + (grow0 + r) * DK + 32 * c;
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        uint32_t ww[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          ww[2 * e] = __float_as_uint(x[4 * h + e].x);
          ww[2 * e + 1] = __float_as_uint(x[4 * h + e].y);
        }
        st_global_v8(dst + 8 * h, ww);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
}

template <int DK, bool DELTA, bool DIAG>
cudaError_t launch_fp32_step(const StepParams& p, cudaStream_t stream);

}  // namespace qs
