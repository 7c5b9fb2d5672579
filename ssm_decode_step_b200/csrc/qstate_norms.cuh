// Per-tile squared Frobenius norms of a stored (quantized) state and of an
// FP32 state, summed in FP64 (qstate_state_sq_norms, qstate_fp32_sq_norms).
// Measurement helpers, not on the decode path: one CTA per tile.
#pragma once

#include "qstate_kernels.cuh"

namespace qs {

constexpr int kNormThreads = 256;

__device__ __forceinline__ double block_sum(double v) {
  __shared__ double part[kNormThreads / 32];
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x < 32) {
    t = threadIdx.x < kNormThreads / 32 ? part[threadIdx.x] : 0.0;
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) t += __shfl_xor_sync(0xffffffffu, t, m);
  }
  return t;
}

// out[tile] = sum of (c * s)^2 over the tile; d = c * s in FP32 as in the
// readout, squared and summed in FP64.
template <int BITS, int DK>
__global__ void __launch_bounds__(kNormThreads) state_sq_norm_kernel(const uint8_t* codes,
                                                                      const float* scales,
                                                                      double* out, int dv,
                                                                      int group) {
  constexpr int LPR = DK / 32;
  constexpr int CW = BITS;
  const size_t tile = blockIdx.x;
  const int ng = DK / group;
  double acc = 0.0;
  for (int rc = threadIdx.x; rc < dv * LPR; rc += kNormThreads) {
    const int r = rc / LPR, c = rc % LPR;
    const size_t row = tile * dv + r;
    const uint4* src = reinterpret_cast<const uint4*>(codes + (row * LPR + c) * (4 * CW));
    uint32_t w[CW];
#pragma unroll
    for (int h = 0; h < CW / 4; ++h) {
      const uint4 u = src[h];
      w[4 * h + 0] = u.x; w[4 * h + 1] = u.y; w[4 * h + 2] = u.z; w[4 * h + 3] = u.w;
    }
    const float s = scales[row * ng + (32 * c) / group];
    float2 d[16];
    decode_chunk<BITS>(w, d);
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const double a = static_cast<double>(__fmul_rn(d[m].x, s));
      const double b = static_cast<double>(__fmul_rn(d[m].y, s));
      acc = __fma_rn(a, a, acc);
      acc = __fma_rn(b, b, acc);
    }
  }
  const double t = block_sum(acc);
  if (threadIdx.x == 0) out[tile] = t;
}

__global__ void __launch_bounds__(kNormThreads) fp32_sq_norm_kernel(const float* S, double* out,
                                                                     long long elems) {
  const float4* src = reinterpret_cast<const float4*>(S + static_cast<size_t>(blockIdx.x) * elems);
  double acc = 0.0;
  for (long long i = threadIdx.x; i < elems / 4; i += kNormThreads) {
    const float4 v = src[i];
    const double a = v.x, b = v.y, c = v.z, d = v.w;
    acc = __fma_rn(a, a, acc);
    acc = __fma_rn(b, b, acc);
    acc = __fma_rn(c, c, acc);
    acc = __fma_rn(d, d, acc);
  }
  const double t = block_sum(acc);
  if (threadIdx.x == 0) out[blockIdx.x] = t;
}

}  // namespace qs
