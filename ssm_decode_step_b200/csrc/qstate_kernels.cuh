// Shared pieces of the quantized-state kernels (sm_100a): the element-level
// arithmetic of the decode step and the quantization-start kernel.  The
// step and readout kernels are in qstate_step.cuh.
//
// The operation (LinQuant eq. (1) with readout o = S q, group-wise INT4/INT8
// state, dynamic / persistent / yoked scales, nearest or Bounded Directional
// Rounding) and its element-level FP32 definition are documented in
// include/qstate.h.
//
// Ownership.  Rows of a tile are independent: every reduction of the step
// (u = S' k, o = x q, the group max) runs along one row.  A thread owns a
// 32-column chunk c of a row (LPR = Dk/32 consecutive lanes per row), so a
// row's reductions are in-thread chains plus log2(LPR) xor shuffles.
//
// Arithmetic.  Each thread holds its chunk as 16 register pairs of adjacent
// columns (2m, 2m+1) and works with the packed FP32 instructions of sm_100
// (__ffma2_rn, __fmul2_rn, __fadd2_rn).  The four packed accumulators of a
// chunk's dot product carry the eight chains of the fixed order (ChunkDot
// below); the lanes of a row then add their chunk sums with xor shuffles 1,
// 2, which is the pairwise tree of the definition.  Every other
// FP32 operation is element-wise, so packed and scalar forms give the same
// bits; explicit rounding intrinsics keep the compiler from contracting or
// reordering (and the library is built -fmad=false).  Codes are unpacked by
// a byte permute into the mantissa of 2^23 (exact) and rounded by adding
// 1.5 * 2^23 inside one fused multiply-add (exact product, ties to even).
//
// No kernel here spins on a flag or barrier: the only waits are
// cp.async.wait_group, __syncthreads and __syncwarp, so nothing can hang.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace qs {

// Threads per CTA.
#ifndef QS_THREADS
#define QS_THREADS 128
#endif
constexpr int kThreads = QS_THREADS;

// Resident CTAs per SM the register allocation targets (kThreads each).
#ifndef QS_MIN_BLOCKS
#define QS_MIN_BLOCKS 4
#endif

// 1.5 * 2^23: adding it to a float of magnitude < 2^22 leaves the nearest
// integer (ties to even) in the low mantissa bits.
constexpr float kMagic = 12582912.0f;

struct StepParams {
  uint8_t* codes;
  float* scales;
  float* shadow;
  const float* q;
  const float* k;
  const float* v;
  const float* alpha;
  const float* beta;
  float* o;
  int tiles;
  int dv;
  int group;
  int rb;              // rows per work unit (divides dv)
  int units_per_tile;  // dv / rb
  int grid_tiles;      // gridDim.x / units_per_tile
  int grid_part;       // gridDim.x % units_per_tile
};

// Work-unit cursor: unit = tile * units_per_tile + part, advanced by gridDim.x
// without a division (the host precomputes the stride's tile / part split).
struct UnitCursor {
  int tile, part;
  __device__ __forceinline__ UnitCursor(int unit, const StepParams& p)
      : tile(unit / p.units_per_tile), part(unit % p.units_per_tile) {}
  __device__ __forceinline__ void advance(const StepParams& p) {
    part += p.grid_part;
    tile += p.grid_tiles;
    if (part >= p.units_per_tile) {
      part -= p.units_per_tile;
      ++tile;
    }
  }
  // first global row of the unit
  __device__ __forceinline__ size_t row0(const StepParams& p) const {
    return static_cast<size_t>(tile) * p.dv + static_cast<size_t>(part) * p.rb;
  }
};

// ---------------------------------------------------------------------------
// small helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}

__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
  unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(s), "l"(gmem) : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may be scheduled while the previous kernel of its stream is
// still running; grid_dep_wait() returns once that kernel has completed and
// its writes are visible, so every such kernel calls it before its first
// global-memory access.  grid_dep_launch() lets the next kernel of the stream
// be scheduled from here on (its CTAs take SM slots as ours retire and wait
// in their own grid_dep_wait()).  Launched without the attribute, both do
// nothing.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
// A hint that brings the line holding p into L2 and nothing into registers.
// It may precede grid_dep_wait(): the loads that use the data come after
// the wait and read L2, where the previous kernel's writes land, so an
// early prefetch can only save their trip to DRAM, never return stale data.
__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];\n" ::"l"(p)); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

template <int N>
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&w)[N]) {
  static_assert(N == 8, "256-bit store takes 8 words");
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"l"(p), "r"(w[0]), "r"(w[1]),
               "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

// ---------------------------------------------------------------------------
// correctly rounded reciprocal and division by qmax
// ---------------------------------------------------------------------------
// Newton-Raphson with a fused correction (Markstein's method): from the
// hardware approximation y of 1/s, e = 1 - s*y is exact in one fused
// multiply-add and y + y*e rounds to 1/s.  Compared bit for bit with the
// IEEE reciprocal on every float in [2^-126, 2^126) (qstate_selfcheck);
// outside that range the IEEE routine is used.
__device__ __forceinline__ float recip_rn(float s) {
  if (s >= 0x1p-126f && s < 0x1p126f) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(s));
    const float e = __fmaf_rn(-s, y, 1.0f);
    return __fmaf_rn(y, e, y);
  }
  return __frcp_rn(s);
}

// m / Q for the constant Q = qmax: the product with RN(1/Q) corrected by the
// exact remainder m - q*Q (division by a constant known in advance, after
// Brisebarre, Muller and Raina).  Compared bit for bit with IEEE division on
// every finite m >= 0 for Q = 7 and Q = 127 (qstate_selfcheck); infinities
// and NaN take the IEEE routine.
template <int Q>
__device__ __forceinline__ float div_qmax_rn(float m) {
  if (m <= 3.40282347e38f) {
    constexpr float r = 1.0f / static_cast<float>(Q);
    const float q0 = __fmul_rn(m, r);
    const float rem = __fmaf_rn(-q0, static_cast<float>(Q), m);
    return __fmaf_rn(rem, r, q0);
  }
  return __fdiv_rn(m, static_cast<float>(Q));
}

// ---------------------------------------------------------------------------
// staged vectors (layout identical on host and device)
// ---------------------------------------------------------------------------

__host__ __device__ __forceinline__ int align_up(int x, int a) { return (x + a - 1) / a * a; }

// Floats per 32-column chunk of a staged vector (32 + 4 padding so that the
// LPR chunks of a row start in different banks).
constexpr int kChunkStride = 36;

// 16-byte unit i of a staged Dk vector lands in chunk i/8 at the padded stride.
__device__ __forceinline__ int vec_unit_offset(int i) { return (i >> 3) * (kChunkStride * 4) + (i & 7) * 16; }

// Load a staged Dk vector's chunk c as 16 pairs (2m, 2m+1).
__device__ __forceinline__ void load_pairs(const unsigned char* base, int c, float2 (&v)[16]) {
  const float4* p4 = reinterpret_cast<const float4*>(base) + c * (kChunkStride / 4);
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const float4 t = p4[m];
    v[2 * m] = make_float2(t.x, t.y);
    v[2 * m + 1] = make_float2(t.z, t.w);
  }
}

// ---------------------------------------------------------------------------
// per-thread decode of a 32-column chunk into pairs e[m] = {c_2m, c_2m+1}
// ---------------------------------------------------------------------------

template <int BITS>
__device__ __forceinline__ void decode_chunk(const uint32_t (&w)[BITS], float2 (&e)[16]) {
  // Offset binary: two's complement code n becomes n + 2^(BITS-1) after
  // flipping the top bit of each field; 0x4B000000 | field is the float
  // 2^23 + field, and subtracting 2^23 + 2^(BITS-1) gives n exactly.
  constexpr float kBias = BITS == 4 ? 8388616.0f : 8388736.0f;
  if constexpr (BITS == 4) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t x = w[q] ^ 0x88888888u;
      const uint32_t lo = x & 0x0F0F0F0Fu;         // columns 8q, 8q+2, 8q+4, 8q+6
      const uint32_t hi = (x >> 4) & 0x0F0F0F0Fu;  // columns 8q+1, 8q+3, 8q+5, 8q+7
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const uint32_t sel = 0x7540u | b;
        e[4 * q + b] = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(lo, 0x4B000000u, sel)),
                                              __uint_as_float(__byte_perm(hi, 0x4B000000u, sel))),
                                  f2(-kBias));
      }
    }
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint32_t x = w[q] ^ 0x80808080u;        // columns 4q .. 4q+3
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        e[2 * q + h] = __fadd2_rn(
            make_float2(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7540u | (2 * h))),
                        __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7540u | (2 * h + 1)))),
            f2(-kBias));
      }
    }
  }
}

// Pack 32 rounded values (floats kMagic + bias + n, as pairs (2m, 2m+1)) into
// BITS words of two's complement codes.
template <int BITS>
__device__ __forceinline__ void pack_chunk(const float2 (&y)[16], uint32_t (&w)[BITS]) {
  if constexpr (BITS == 4) {
    // Low 4 bits of each value are n + 8 in 1..15; (odd << 4) + even has the
    // byte (n_odd + 8, n_even + 8) in its low 8 bits with no carry.
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t by[4];
#pragma unroll
      for (int b = 0; b < 4; ++b)
        by[b] = (__float_as_uint(y[4 * q + b].y) << 4) + __float_as_uint(y[4 * q + b].x);
      const uint32_t t0 = __byte_perm(by[0], by[1], 0x0040u);
      const uint32_t t1 = __byte_perm(by[2], by[3], 0x0040u);
      w[q] = __byte_perm(t0, t1, 0x5410u) ^ 0x88888888u;
    }
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint32_t t0 = __byte_perm(__float_as_uint(y[2 * q].x), __float_as_uint(y[2 * q].y), 0x0040u);
      const uint32_t t1 =
          __byte_perm(__float_as_uint(y[2 * q + 1].x), __float_as_uint(y[2 * q + 1].y), 0x0040u);
      w[q] = __byte_perm(t0, t1, 0x5410u) ^ 0x80808080u;
    }
  }
}

// The fixed dot-product order within a 32-column chunk held as 16 register
// pairs (2m, 2m+1): eight fused multiply-add chains from +0, chain r over
// the columns r, r + 8, r + 16, r + 24 in that order.  Pair m carries the
// columns 2m and 2m + 1, so packed accumulator p[m & 3] holds the chains
// (2(m & 3), 2(m & 3) + 1), and feeding the pairs in ascending m keeps every
// chain in column order.  The chunk sum is ((c0 + c4) + (c2 + c6)) +
// ((c1 + c5) + (c3 + c7)).
struct ChunkDot {
  float2 p[4];
  __device__ __forceinline__ ChunkDot() {
#pragma unroll
    for (int i = 0; i < 4; ++i) p[i] = make_float2(0.0f, 0.0f);
  }
  __device__ __forceinline__ void add(int m, float2 a, float2 b) { p[m & 3] = __ffma2_rn(a, b, p[m & 3]); }
  __device__ __forceinline__ float sum() const {
    const float2 q = __fadd2_rn(__fadd2_rn(p[0], p[2]), __fadd2_rn(p[1], p[3]));
    return __fadd_rn(q.x, q.y);
  }
};

// The whole chunk a . b in the fixed order.
__device__ __forceinline__ float chunk_sum(const float2 (&a)[16], const float2 (&b)[16]) {
  ChunkDot d;
#pragma unroll
  for (int m = 0; m < 16; ++m) d.add(m, a[m], b[m]);
  return d.sum();
}

// The chunk sums of a row's LPR lanes combined by the pairwise tree (xor 1,
// then xor 2): ((c0 + c1) + (c2 + c3)); every lane of the row gets the same
// bits because each addition is commutative.
template <int LPR>
__device__ __forceinline__ float row_tree(float t) {
#pragma unroll
  for (int m = 1; m < LPR; m <<= 1) t = __fadd_rn(t, __shfl_xor_sync(0xffffffffu, t, m));
  return t;
}

template <int LPR>
__device__ __forceinline__ float row_max(float m, int group) {
  // group / 32 lanes share a quantization group
  if (group >= 64) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
  if (group >= 128 && LPR >= 4) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
  return m;
}

__device__ __forceinline__ float chunk_absmax(const float2 (&x)[16]) {
  float m0 = 0.0f, m1 = 0.0f;
#pragma unroll
  for (int m = 0; m < 16; m += 2) {
    m0 = fmaxf(m0, fmaxf(fabsf(x[m].x), fabsf(x[m].y)));
    m1 = fmaxf(m1, fmaxf(fabsf(x[m + 1].x), fabsf(x[m + 1].y)));
  }
  return fmaxf(m0, m1);
}

// Round x * inv to the grid (nearest, ties to even, exact product), with the
// result held as the float kMagic + bias + n.  `clamp` selects the general
// path that also bounds n to [-qmax, qmax] (and handles huge products).
template <int BITS>
__device__ __forceinline__ void round_chunk(const float2 (&x)[16], float inv, bool clamp,
                                            float2 (&y)[16]) {
  constexpr float kOff = kMagic + (BITS == 4 ? 8.0f : 128.0f);
  constexpr float kQ = BITS == 4 ? 7.0f : 127.0f;
#pragma unroll
  for (int m = 0; m < 16; ++m) y[m] = __ffma2_rn(x[m], f2(inv), f2(kOff));
  if (clamp) {
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      y[m].x = fminf(fmaxf(y[m].x, kOff - kQ), kOff + kQ);
      y[m].y = fminf(fmaxf(y[m].y, kOff - kQ), kOff + kQ);
    }
  }
}

// Bounded Directional Rounding on rounded values y (see qstate.h): with
// sigma = sign(w) sign(k_j), move n one step toward the update when n*s'
// lies on the wrong side of d, the element as stored before the step.
template <int BITS>
__device__ __forceinline__ void bdr_chunk(float2 (&y)[16], const float2 (&d)[16],
                                          const float2 (&sk)[16], float sw, float sp) {
  constexpr float kOff = kMagic + (BITS == 4 ? 8.0f : 128.0f);
  constexpr float kQ = BITS == 4 ? 7.0f : 127.0f;
  float hi = kOff, lo = kOff;
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    // reversed iff sigma (n s') < sigma d; the products by sigma in
    // {-1, 0, 1} are exact, and comparing the two rounded values directly
    // (no subtraction after the product) leaves nothing to contract
    const float2 nf = __fadd2_rn(y[m], f2(-kOff));   // n, exact
    const float2 dq = __fmul2_rn(nf, f2(sp));        // n * s'
    const float2 sg = __fmul2_rn(sk[m], f2(sw));     // sigma
    const float2 a = __fmul2_rn(dq, sg);
    const float2 b = __fmul2_rn(d[m], sg);
    const float yx = a.x < b.x ? __fadd_rn(y[m].x, sg.x) : y[m].x;
    const float yy = a.y < b.y ? __fadd_rn(y[m].y, sg.y) : y[m].y;
    y[m].x = yx;
    y[m].y = yy;
    hi = fmaxf(hi, fmaxf(yx, yy));
    lo = fminf(lo, fminf(yx, yy));
  }
  // only a moved code can leave [-qmax, qmax]: clamp when the extremes show one did
  if (hi > kOff + kQ || lo < kOff - kQ) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      y[i].x = fminf(fmaxf(y[i].x, kOff - kQ), kOff + kQ);
      y[i].y = fminf(fmaxf(y[i].y, kOff - kQ), kOff + kQ);
    }
  }
}

// ---------------------------------------------------------------------------
// quantization start: S0 -> codes, scales (dynamic rule, nearest); shadow copy
// ---------------------------------------------------------------------------
template <int BITS, int DK>
__global__ void __launch_bounds__(256) init_kernel(const float* __restrict__ S0, uint8_t* codes,
                                                   float* scales, float* shadow, long long rows,
                                                   int group) {
  constexpr int LPR = DK / 32;
  constexpr int CW = BITS;
  constexpr int QMAX = BITS == 4 ? 7 : 127;
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long rowg = gid / LPR;
  const int c = static_cast<int>(gid % LPR);
  const bool active = rowg < rows;  // whole warps stay for the shuffles
  float2 x[16];
  const float4* src = reinterpret_cast<const float4*>(S0 + (active ? rowg : 0) * DK + 32 * c);
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const float4 t = src[u];
    x[2 * u] = make_float2(t.x, t.y);
    x[2 * u + 1] = make_float2(t.z, t.w);
  }
  const float s = div_qmax_rn<QMAX>(row_max<LPR>(chunk_absmax(x), group));
  uint32_t out[CW];
  if (s > 0.0f) {
    const float inv = recip_rn(s);
    const bool clamp = !(s >= 0x1p-126f && s < 0x1p126f);
    float2 y[16];
    round_chunk<BITS>(x, inv, clamp, y);
    pack_chunk<BITS>(y, out);
  } else {
#pragma unroll
    for (int q = 0; q < CW; ++q) out[q] = 0u;
  }
  if (!active) return;
  uint8_t* cg = codes + (rowg * LPR + c) * (4 * CW);
  if constexpr (CW == 4) {
    *reinterpret_cast<uint4*>(cg) = make_uint4(out[0], out[1], out[2], out[3]);
  } else {
    st_global_v8(cg, out);
  }
  const int ng = DK / group, g = (32 * c) / group;
  if ((32 * c) % group == 0) scales[rowg * ng + g] = s;
  if (shadow != nullptr) {
    float4* dst = reinterpret_cast<float4*>(shadow + rowg * DK + 32 * c);
#pragma unroll
    for (int u = 0; u < 8; ++u) dst[u] = make_float4(x[2 * u].x, x[2 * u].y, x[2 * u + 1].x, x[2 * u + 1].y);
  }
}

}  // namespace qs
