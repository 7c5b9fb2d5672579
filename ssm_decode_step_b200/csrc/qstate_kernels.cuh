// Fused decode-step kernels for the quantized recurrent state (sm_100a).
//
// The operation (LinQuant eq. (1) with readout o = S q, group-wise INT4/INT8
// state, dynamic / persistent / yoked scales, nearest or Bounded Directional
// Rounding) and its element-level FP32 definition are documented in
// include/qstate.h.  This file is the CUDA realization of that definition.
//
// Work decomposition.  Rows of a tile are independent: every reduction of
// the step (u = S' k, o = x q, the group max) runs along one row.  A thread
// owns a 32-column chunk of one row (LPR = Dk/32 lanes per row, consecutive
// lanes), so the row's reductions are in-thread chains plus log2(LPR) xor
// shuffles.  A CTA owns one tile at a time (blockDim = Dv * LPR threads) and
// walks tiles with a stride of gridDim.x (persistent grid, sized to the SMs).
//
// Memory path.  Each tile's codes, scales, v, k, q (and alpha, the FP32
// shadow) are staged into shared memory with cp.async through an S-deep
// ring, so S-1 tiles are in flight while one is computed.  k, q and a
// diagonal alpha are scattered into a pair-interleaved layout (column m and
// m+16 of a chunk side by side) so the packed FP32 instructions
// (__ffma2_rn & co., sm_100) see their operands in register pairs.  New codes
// leave as 16/32-byte coalesced stores straight from registers.
//
// Order of FP32 operations.  Each thread evaluates its chunk's two 16-column
// segments as two fused multiply-add chains in column order (the two lanes
// of one packed instruction), adds the pair, then the lanes of the row add
// their partials with xor shuffles 1, 2: exactly the balanced pairwise tree
// over 16-column segments that the definition fixes.  Every other FP32
// operation is element-wise, so packed and scalar forms give the same bits.
// Explicit intrinsics (__fmul_rn, __fadd_rn, __ffma2_rn ...) keep the compiler
// from contracting or reordering; the library is also built -fmad=false.
//
// No kernel here spins on a flag or barrier: the only waits are
// cp.async.wait_group and __syncthreads, so nothing can hang.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace qs {

constexpr int kMaxThreads = 512;

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

__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

__device__ __forceinline__ float2 abs2(float2 a) { return make_float2(fabsf(a.x), fabsf(a.y)); }

template <int N>
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&w)[N]) {
  static_assert(N == 8, "256-bit store takes 8 words");
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"l"(p), "r"(w[0]), "r"(w[1]),
               "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

// Position of column r (0..31) of a chunk in the pair-interleaved layout:
// columns m and m+16 sit side by side.
__host__ __device__ __forceinline__ int pair_pos(int r) { return r < 16 ? 2 * r : 2 * (r - 16) + 1; }

// Floats per interleaved chunk in shared memory (32 + 4 padding so that the
// LPR chunks of a row start in different banks).
constexpr int kChunkStride = 36;

// ---------------------------------------------------------------------------
// shared-memory stage layout (identical on host and device)
// ---------------------------------------------------------------------------

__host__ __device__ __forceinline__ int align_up(int x, int a) { return (x + a - 1) / a * a; }

struct StageLayout {
  int codes, scales, v, k, q, a, sk, misc, shadow, bytes;

  __host__ __device__ StageLayout(int bits, int dk, int dv, int group, bool diag, bool bdr,
                                  bool yoked) {
    const int vec = (dk / 32) * kChunkStride * 4;
    int off = 0;
    codes = off;  off = align_up(off + dv * dk * bits / 8, 16);
    scales = off; off = align_up(off + dv * (dk / group) * 4, 16);
    v = off;      off = align_up(off + dv * 4, 16);
    k = off;      off += vec;
    q = off;      off += vec;
    a = off;      off += diag ? vec : 0;
    sk = off;     off += bdr ? vec : 0;
    misc = off;   off += 16;
    shadow = off; off += yoked ? dv * dk * 4 : 0;
    bytes = align_up(off, 128);
  }
};

// Issue the cp.async copies of one tile into a stage.
template <int BITS, int DK, bool DIAG, bool YOKED, bool WITH_STATE_UPDATE>
__device__ __forceinline__ void stage_load(unsigned char* st, const StageLayout& L,
                                           const StepParams& p, int tile) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int dv = p.dv;
  const size_t t = static_cast<size_t>(tile);
  {
    const int n16 = dv * DK * BITS / 8 / 16;
    const uint8_t* g = p.codes + t * (dv * DK * BITS / 8);
    for (int i = tid; i < n16; i += nt) cp_async16(st + L.codes + 16 * i, g + 16 * i);
  }
  {
    const int n16 = dv * (DK / p.group) * 4 / 16;
    const float* g = p.scales + t * (dv * (DK / p.group));
    for (int i = tid; i < n16; i += nt) cp_async16(st + L.scales + 16 * i, g + 4 * i);
  }
  float* sk = reinterpret_cast<float*>(st + L.k);
  float* sq = reinterpret_cast<float*>(st + L.q);
  for (int j = tid; j < DK; j += nt) {
    const int pos = (j / 32) * kChunkStride + pair_pos(j % 32);
    if (p.o != nullptr) cp_async4(sq + pos, p.q + t * DK + j);
    if constexpr (WITH_STATE_UPDATE) {
      cp_async4(sk + pos, p.k + t * DK + j);
      if constexpr (DIAG) cp_async4(reinterpret_cast<float*>(st + L.a) + pos, p.alpha + t * DK + j);
    }
  }
  if constexpr (WITH_STATE_UPDATE) {
    const int n16 = dv * 4 / 16;
    for (int i = tid; i < n16; i += nt) cp_async16(st + L.v + 16 * i, p.v + t * dv + 4 * i);
    if (tid == 0) {
      float* misc = reinterpret_cast<float*>(st + L.misc);
      if constexpr (!DIAG) cp_async4(misc + 0, p.alpha + t);
      cp_async4(misc + 1, p.beta + t);
    }
  }
  if constexpr (YOKED) {
    // 16-byte unit u of row-chunk rc lands at unit position u ^ (rc & 7) so
    // that the 8 lanes of a quarter-warp read 8 different bank groups.
    const int n16 = dv * DK / 4;
    const float* g = p.shadow + t * (dv * DK);
    for (int i = tid; i < n16; i += nt) {
      const int rc = i >> 3, u = i & 7;
      cp_async16(st + L.shadow + rc * 128 + 16 * (u ^ (rc & 7)), g + 4 * i);
    }
  }
}

// ---------------------------------------------------------------------------
// per-thread decode of a 32-column chunk into pairs e[m] = {c_m, c_{m+16}}
// ---------------------------------------------------------------------------

template <int BITS>
__device__ __forceinline__ void decode_chunk(const uint32_t (&w)[BITS], float2 (&e)[16]) {
  // Offset binary: two's complement code n becomes n + 2^(BITS-1) after
  // flipping the top bit of each field; 0x4B000000 | field is the float
  // 2^23 + field, and subtracting 2^23 + 2^(BITS-1) gives n exactly.
  constexpr float kBias = BITS == 4 ? 8388616.0f : 8388736.0f;
  if constexpr (BITS == 4) {
    uint32_t lo[4], hi[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t x = w[q] ^ 0x88888888u;
      lo[q] = x & 0x0F0F0F0Fu;         // nibbles 0,2,4,6 of the word
      hi[q] = (x >> 4) & 0x0F0F0F0Fu;  // nibbles 1,3,5,7
    }
    // element 8q + 2b -> byte b of lo[q]; element 8q + 2b + 1 -> byte b of hi[q]
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const int qa = m / 8, qb = 2 + m / 8, nib = m % 8;
      const uint32_t sa = (nib & 1) ? hi[qa] : lo[qa];
      const uint32_t sb = (nib & 1) ? hi[qb] : lo[qb];
      const uint32_t sel = 0x7540u | (nib >> 1);
      const float fa = __uint_as_float(__byte_perm(sa, 0x4B000000u, sel));
      const float fb = __uint_as_float(__byte_perm(sb, 0x4B000000u, sel));
      e[m] = __fadd2_rn(make_float2(fa, fb), f2(-kBias));
    }
  } else {
    uint32_t x[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) x[q] = w[q] ^ 0x80808080u;
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const int qa = m / 4, qb = 4 + m / 4, b = m % 4;
      const uint32_t sel = 0x7540u | b;
      const float fa = __uint_as_float(__byte_perm(x[qa], 0x4B000000u, sel));
      const float fb = __uint_as_float(__byte_perm(x[qb], 0x4B000000u, sel));
      e[m] = __fadd2_rn(make_float2(fa, fb), f2(-kBias));
    }
  }
}

// Pack 32 rounded values (held as kMagic + bias + n floats in pairs) into
// BITS words of two's complement codes.
template <int BITS>
__device__ __forceinline__ void pack_chunk(const float2 (&y)[16], uint32_t (&w)[BITS]) {
  auto Y = [&](int e) -> uint32_t {
    return __float_as_uint(e < 16 ? y[e].x : y[e - 16].y);
  };
  if constexpr (BITS == 4) {
    // Low 4 bits of each value are n + 8 in 1..15; (b << 4) + a has the byte
    // (n_b + 8, n_a + 8) in its low 8 bits with no carry.
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t by[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int e = 8 * q + 2 * b;
        by[b] = (Y(e + 1) << 4) + Y(e);
      }
      const uint32_t t0 = __byte_perm(by[0], by[1], 0x0040u);
      const uint32_t t1 = __byte_perm(by[2], by[3], 0x0040u);
      w[q] = __byte_perm(t0, t1, 0x5410u) ^ 0x88888888u;
    }
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint32_t t0 = __byte_perm(Y(4 * q), Y(4 * q + 1), 0x0040u);
      const uint32_t t1 = __byte_perm(Y(4 * q + 2), Y(4 * q + 3), 0x0040u);
      w[q] = __byte_perm(t0, t1, 0x5410u) ^ 0x80808080u;
    }
  }
}

// Sum of the chunk's two segment chains, then the pairwise tree across the
// LPR lanes of the row (xor 1, then xor 2).
template <int LPR>
__device__ __forceinline__ float row_tree(float2 acc) {
  float t = __fadd_rn(acc.x, acc.y);
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
// lies on the wrong side of the pre-update value S'.
template <int BITS>
__device__ __forceinline__ void bdr_chunk(float2 (&y)[16], const float2 (&Sp)[16],
                                          const float2* sk, float sw, float sp) {
  constexpr float kOff = kMagic + (BITS == 4 ? 8.0f : 128.0f);
  constexpr float kQ = BITS == 4 ? 7.0f : 127.0f;
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    const float2 nf = __fadd2_rn(y[m], f2(-kOff));          // n, exact
    const float2 dq = __fmul2_rn(nf, f2(sp));               // n * s'
    const float2 e = __fadd2_rn(Sp[m], make_float2(-dq.x, -dq.y));  // sign of S' - n s'
    const float2 sg = __fmul2_rn(sk[m], f2(sw));            // sigma in {-1, 0, 1}
    const float2 t = __fmul2_rn(e, sg);                      // > 0 iff reversed
    float yx = t.x > 0.0f ? __fadd_rn(y[m].x, sg.x) : y[m].x;
    float yy = t.y > 0.0f ? __fadd_rn(y[m].y, sg.y) : y[m].y;
    y[m].x = fminf(fmaxf(yx, kOff - kQ), kOff + kQ);
    y[m].y = fminf(fmaxf(yy, kOff - kQ), kOff + kQ);
  }
}

// ---------------------------------------------------------------------------
// the decode step
// ---------------------------------------------------------------------------
// POLICY: 0 dynamic, 1 persistent, 2 yoked.
template <int BITS, int DK, int POLICY, bool BDR, bool DELTA, bool DIAG, int STAGES>
__global__ void __launch_bounds__(kMaxThreads, 1) step_kernel(StepParams p) {
  constexpr int LPR = DK / 32;
  constexpr bool YOKED = POLICY == 2;
  constexpr int CW = BITS;  // 32-bit words of codes per 32-column chunk
  constexpr float kQf = BITS == 4 ? 7.0f : 127.0f;
  constexpr float kOff = kMagic + (BITS == 4 ? 8.0f : 128.0f);

  extern __shared__ __align__(128) unsigned char smem[];
  const StageLayout L(BITS, DK, p.dv, p.group, DIAG, BDR, YOKED);
  const int tid = threadIdx.x;
  const int row = tid / LPR, c = tid % LPR;
  const int ng = DK / p.group;
  const int g = (32 * c) / p.group;
  const bool readout = p.o != nullptr;

  // prologue: STAGES-1 tiles in flight
#pragma unroll
  for (int s = 0; s < STAGES - 1; ++s) {
    const int tile = blockIdx.x + s * gridDim.x;
    if (tile < p.tiles) stage_load<BITS, DK, DIAG, YOKED, true>(smem + s * L.bytes, L, p, tile);
    cp_async_commit();
  }

  int it = 0;
  for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++it) {
    {
      const int pre = tile + (STAGES - 1) * gridDim.x;
      if (pre < p.tiles)
        stage_load<BITS, DK, DIAG, YOKED, true>(smem + ((it + STAGES - 1) % STAGES) * L.bytes, L, p,
                                                pre);
      cp_async_commit();
    }
    cp_async_wait<STAGES - 1>();
    __syncthreads();
    unsigned char* st = smem + (it % STAGES) * L.bytes;

    if constexpr (BDR) {
      // sign(k_j) per column, same interleaved layout as k
      const float* kvals = reinterpret_cast<const float*>(st + L.k);
      float* ss = reinterpret_cast<float*>(st + L.sk);
      for (int j = tid; j < DK; j += blockDim.x) {
        const int pos = (j / 32) * kChunkStride + pair_pos(j % 32);
        const float kv = kvals[pos];
        ss[pos] = kv > 0.0f ? 1.0f : (kv < 0.0f ? -1.0f : 0.0f);
      }
      __syncthreads();
    }

    // ---- a1: load and unpack this thread's 32 codes
    uint32_t w[CW];
    {
      const uint4* src = reinterpret_cast<const uint4*>(st + L.codes + (row * LPR + c) * (4 * CW));
#pragma unroll
      for (int q = 0; q < CW / 4; ++q) {
        const uint4 u = src[q];
        w[4 * q + 0] = u.x; w[4 * q + 1] = u.y; w[4 * q + 2] = u.z; w[4 * q + 3] = u.w;
      }
    }
    const float s_old = reinterpret_cast<const float*>(st + L.scales)[row * ng + g];
    const float* miscf = reinterpret_cast<const float*>(st + L.misc);
    const float beta = miscf[1];
    const float v_i = reinterpret_cast<const float*>(st + L.v)[row];
    const float2* kp = reinterpret_cast<const float2*>(st + L.k) + c * (kChunkStride / 2);
    float2 kk[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) kk[m] = kp[m];

    // ---- a2: dequantize and decay
    float2 Sp[16];
    decode_chunk<BITS>(w, Sp);
    if constexpr (DIAG) {
      const float2* ap = reinterpret_cast<const float2*>(st + L.a) + c * (kChunkStride / 2);
#pragma unroll
      for (int m = 0; m < 16; ++m) Sp[m] = __fmul2_rn(__fmul2_rn(Sp[m], f2(s_old)), ap[m]);
    } else {
      const float a = miscf[0];
#pragma unroll
      for (int m = 0; m < 16; ++m) Sp[m] = __fmul2_rn(__fmul2_rn(Sp[m], f2(s_old)), f2(a));
    }

    // ---- a3/a4: key projection and rank-1 write
    float wcoef;
    if constexpr (DELTA) {
      float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int m = 0; m < 16; ++m) acc = __ffma2_rn(Sp[m], kk[m], acc);
      const float u = row_tree<LPR>(acc);
      wcoef = __fmul_rn(beta, __fsub_rn(v_i, u));
    } else {
      wcoef = __fmul_rn(beta, v_i);
    }
    float2 x[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) x[m] = __ffma2_rn(f2(wcoef), kk[m], Sp[m]);

    // ---- a5: readout from the updated state
    if (readout) {
      const float2* qp = reinterpret_cast<const float2*>(st + L.q) + c * (kChunkStride / 2);
      float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int m = 0; m < 16; ++m) acc = __ffma2_rn(x[m], qp[m], acc);
      const float o = row_tree<LPR>(acc);
      if (c == 0) p.o[static_cast<size_t>(tile) * p.dv + row] = o;
    }

    // ---- a6/a7: scale selection (yoked shadow update)
    float sp;
    if constexpr (POLICY == 0) {
      const float m = row_max<LPR>(chunk_absmax(x), p.group);
      sp = __fdiv_rn(m, kQf);
    } else if constexpr (POLICY == 1) {
      sp = s_old;
    } else {
      // shadow chunk from shared memory (swizzled 16-byte units)
      const int rc = row * LPR + c;
      const float4* rs = reinterpret_cast<const float4*>(st + L.shadow + rc * 128);
      float r[32];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float4 t = rs[u ^ (rc & 7)];
        r[4 * u] = t.x; r[4 * u + 1] = t.y; r[4 * u + 2] = t.z; r[4 * u + 3] = t.w;
      }
      // R' = R * a
      if constexpr (DIAG) {
        const float* ap = reinterpret_cast<const float*>(st + L.a) + c * kChunkStride;
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = __fmul_rn(r[j], ap[pair_pos(j)]);
      } else {
        const float a = miscf[0];
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = __fmul_rn(r[j], a);
      }
      float wr;
      if constexpr (DELTA) {
        float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          a0 = __fmaf_rn(r[j], kk[j].x, a0);
          a1 = __fmaf_rn(r[16 + j], kk[j].y, a1);
        }
        const float ur = row_tree<LPR>(make_float2(a0, a1));
        wr = __fmul_rn(beta, __fsub_rn(v_i, ur));
      } else {
        wr = wcoef;
      }
      float mr = 0.0f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        r[j] = __fmaf_rn(wr, kk[j].x, r[j]);
        r[16 + j] = __fmaf_rn(wr, kk[j].y, r[16 + j]);
        mr = fmaxf(mr, fmaxf(fabsf(r[j]), fabsf(r[16 + j])));
      }
      float* rg = p.shadow + static_cast<size_t>(tile) * p.dv * DK + row * DK + 32 * c;
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        uint32_t ww[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) ww[e] = __float_as_uint(r[8 * h + e]);
        st_global_v8(rg + 8 * h, ww);
      }
      mr = row_max<LPR>(mr, p.group);
      sp = __fdiv_rn(mr, kQf);
    }

    // ---- a8: round (and BDR)
    uint32_t out[CW];
    if (sp > 0.0f) {
      const float inv = __frcp_rn(sp);
      bool clamp;
      if constexpr (POLICY == 0) {
        // |x| <= group max, so |x * inv| <= qmax(1 + 2^-23) rounds inside the
        // range unless the scale is not a normal finite float
        clamp = !(sp >= 1.17549435e-38f && sp <= 3.40282347e38f);
      } else {
        const float xm = chunk_absmax(x);
        clamp = !(__fmaf_rn(xm, inv, kOff) <= kOff + kQf);
      }
      float2 y[16];
      round_chunk<BITS>(x, inv, clamp, y);
      if constexpr (BDR) {
        const float2* skp = reinterpret_cast<const float2*>(st + L.sk) + c * (kChunkStride / 2);
        const float sw = wcoef > 0.0f ? 1.0f : (wcoef < 0.0f ? -1.0f : 0.0f);
        bdr_chunk<BITS>(y, Sp, skp, sw, sp);
      }
      pack_chunk<BITS>(y, out);
    } else {
#pragma unroll
      for (int q = 0; q < CW; ++q) out[q] = 0u;
    }

    // ---- a9: store codes (and scales)
    uint8_t* cg = p.codes + static_cast<size_t>(tile) * p.dv * DK * BITS / 8 + (row * LPR + c) * (4 * CW);
    if constexpr (CW == 4) {
      *reinterpret_cast<uint4*>(cg) = make_uint4(out[0], out[1], out[2], out[3]);
    } else {
      st_global_v8(cg, out);
    }
    if constexpr (POLICY != 1) {
      if ((32 * c) % p.group == 0) p.scales[(static_cast<size_t>(tile) * p.dv + row) * ng + g] = sp;
    }
    __syncthreads();
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// readout of the stored state (no update)
// ---------------------------------------------------------------------------
template <int BITS, int DK, int STAGES>
__global__ void __launch_bounds__(kMaxThreads, 1) readout_kernel(StepParams p) {
  constexpr int LPR = DK / 32;
  constexpr int CW = BITS;
  extern __shared__ __align__(128) unsigned char smem[];
  const StageLayout L(BITS, DK, p.dv, p.group, false, false, false);
  const int tid = threadIdx.x;
  const int row = tid / LPR, c = tid % LPR;
  const int ng = DK / p.group;
  const int g = (32 * c) / p.group;

#pragma unroll
  for (int s = 0; s < STAGES - 1; ++s) {
    const int tile = blockIdx.x + s * gridDim.x;
    if (tile < p.tiles) stage_load<BITS, DK, false, false, false>(smem + s * L.bytes, L, p, tile);
    cp_async_commit();
  }
  int it = 0;
  for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++it) {
    {
      const int pre = tile + (STAGES - 1) * gridDim.x;
      if (pre < p.tiles)
        stage_load<BITS, DK, false, false, false>(smem + ((it + STAGES - 1) % STAGES) * L.bytes, L,
                                                  p, pre);
      cp_async_commit();
    }
    cp_async_wait<STAGES - 1>();
    __syncthreads();
    unsigned char* st = smem + (it % STAGES) * L.bytes;
    uint32_t w[CW];
    const uint4* src = reinterpret_cast<const uint4*>(st + L.codes + (row * LPR + c) * (4 * CW));
#pragma unroll
    for (int q = 0; q < CW / 4; ++q) {
      const uint4 u = src[q];
      w[4 * q + 0] = u.x; w[4 * q + 1] = u.y; w[4 * q + 2] = u.z; w[4 * q + 3] = u.w;
    }
    const float s = reinterpret_cast<const float*>(st + L.scales)[row * ng + g];
    float2 d[16];
    decode_chunk<BITS>(w, d);
    const float2* qp = reinterpret_cast<const float2*>(st + L.q) + c * (kChunkStride / 2);
    float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int m = 0; m < 16; ++m) acc = __ffma2_rn(__fmul2_rn(d[m], f2(s)), qp[m], acc);
    const float o = row_tree<LPR>(acc);
    if (c == 0) p.o[static_cast<size_t>(tile) * p.dv + row] = o;
    __syncthreads();
  }
  cp_async_wait<0>();
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
  constexpr float kQf = BITS == 4 ? 7.0f : 127.0f;
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long rowg = gid / LPR;
  const int c = static_cast<int>(gid % LPR);
  const bool active = rowg < rows;  // whole warps stay for the shuffles
  float r[32];
  const float* src = S0 + (active ? rowg : 0) * DK + 32 * c;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const float4 t = reinterpret_cast<const float4*>(src)[u];
    r[4 * u] = t.x; r[4 * u + 1] = t.y; r[4 * u + 2] = t.z; r[4 * u + 3] = t.w;
  }
  float2 x[16];
#pragma unroll
  for (int m = 0; m < 16; ++m) x[m] = make_float2(r[m], r[16 + m]);
  const float m = row_max<LPR>(chunk_absmax(x), group);
  const float s = __fdiv_rn(m, kQf);
  uint32_t out[CW];
  if (s > 0.0f) {
    const float inv = __frcp_rn(s);
    const bool clamp = !(s >= 1.17549435e-38f && s <= 3.40282347e38f);
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
    float* dst = shadow + rowg * DK + 32 * c;
#pragma unroll
    for (int u = 0; u < 8; ++u)
      reinterpret_cast<float4*>(dst)[u] = make_float4(r[4 * u], r[4 * u + 1], r[4 * u + 2], r[4 * u + 3]);
  }
}

}  // namespace qs
