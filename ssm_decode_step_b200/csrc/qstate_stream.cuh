// The decode step for the dynamic and persistent scale policies, with the
// state streamed through registers (sm_100a).
//
// Work decomposition (as the ring kernel of qstate_step.cuh): a row block is
// RW = 32 / (Dk/32) consecutive rows of one tile; lane (rr, c) of a warp owns
// the 32-column chunk c of row rr, so every reduction of the step is an
// in-lane chain plus log2(Dk/32) xor shuffles.  The row blocks of all tiles
// form one sequence cut into one contiguous range per warp.  One warp per
// CTA; nothing waits for another warp.
//
// Memory path.  A row block's codes are one contiguous run of RW * Dk *
// bits / 8 bytes, and lane l's chunk is its l-th 16-byte (INT4) or 32-byte
// (INT8) unit; its scales and v are contiguous too.  Each lane loads its
// codes, its group's scale and its row's v straight into registers with one
// 128- or 256-bit load and two 32-bit loads, two row blocks ahead of their
// use: the loop alternates two register sets, and a set is refilled as soon
// as its codes are unpacked.  No shared memory, copy or barrier sits on the
// state's path.  The per-tile vectors (k, q, diagonal alpha, alpha, beta)
// go by cp.async into one of two per-warp shared-memory slots a tile ahead;
// k lives in registers for the tile (or, for the BDR instances, is re-read
// from the slot at each use), q and diagonal alpha are read from the slot.
// New codes, scales and o leave straight from registers.
//
// Element arithmetic (the definition of include/qstate.h, fixed order):
//   unpack     INT4: one LOP3 per element builds the float 2^23 + 16^p (c+8)
//              from nibble p of the word (or of the word shifted down by 16),
//              and one packed fused multiply-add per pair scales by 16^-p
//              and removes the offset: exactly c.  INT8: byte permutes into
//              the mantissa of 2^23 and one packed add.
//   dequantize S' = c * (s * a_j)
//   write      w = beta (v - u), u = S' . k (delta = 1); x = fused(w k_j + S')
//   readout    o = x . q
//   scale      dynamic: max |x| / qmax; persistent: s
//   round      fused(x * (1/s') + 1.5 * 2^23 + 2^(bits-1)): the exact product
//              rounded to an integer, held in the low mantissa bits as the
//              offset-binary code; persistent scales clamp every element
//              (the lower side by a min/max, the upper by the saturating
//              pack)
//   BDR        persistent: on the packed words (below); dynamic: the
//              dequantized comparison of qstate_kernels.cuh
//   pack       dynamic: offset-binary fields to two's complement words;
//              persistent: saturating integer packs
#pragma once

#include "qstate_kernels.cuh"

namespace qs {

// Registers per thread of the streamed step: 128 leaves room for 16 resident
// warps per SM; BDR instances hold the stored codes and the update-sign
// masks as well and get 168, the most that still leaves 12 warps per SM
// (65536 / (168 x 32) = 12.2), INT8 ones (twice the words) 200.
#ifndef QS_STREAM_REGS
#define QS_STREAM_REGS 128
#endif
#ifndef QS_STREAM_REGS_BDR
#define QS_STREAM_REGS_BDR 168
#endif
#ifndef QS_STREAM_REGS_BDR8
#define QS_STREAM_REGS_BDR8 200
#endif
// Where the tile's key vector lives: 1 reads it from its shared-memory slot
// at each use, 0 holds it in registers for the tile, -1 (default) does the
// former for the BDR instances (whose packed-word masks and stored codes
// take registers of their own) and the latter for the others.
#ifndef QS_STREAM_K_SMEM
#define QS_STREAM_K_SMEM -1
#endif

struct StreamParams {
  uint8_t* codes;
  float* scales;
  const float* q;
  const float* k;
  const float* v;
  const float* alpha;
  const float* beta;
  float* o;
  int nblocks;  // row blocks in all tiles: tiles * dv / RW
  int bpt;      // row blocks per tile: dv / RW
  int group;
  // the bits of the float 2^23 (0x4B000000), passed at run time so that the
  // INT4 unpack keeps it in one register and merges each field into it with
  // a single logic operation
  uint32_t two23;
};

// One warp's shared memory: two tile-vector slots (k, q, diagonal alpha and,
// for BDR under a changing scale, sign(k) at the padded chunk stride; then
// alpha and beta).
struct StreamLayout {
  int k, q, a, sk, misc, slot;
  __host__ __device__ StreamLayout(int dk, bool diag, bool sign_k) {
    const int vec = (dk / 32) * kChunkStride * 4;
    int off = 0;
    k = off;    off += vec;
    q = off;    off += vec;
    a = off;    off += diag ? vec : 0;
    sk = off;   off += sign_k ? vec : 0;
    misc = off; off += 16;
    slot = align_up(off, 128);
  }
  __host__ __device__ int bytes() const { return 2 * slot; }
};

// A staged Dk vector's chunk c as 16 pairs, re-read from shared memory at
// every call (volatile: the compiler may not keep an earlier read instead).
__device__ __forceinline__ void load_pairs_v(const unsigned char* base, int c, float2 (&v)[16]) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(base)) + c * (kChunkStride * 4);
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    float4 t;
    asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];\n"
                 : "=f"(t.x), "=f"(t.y), "=f"(t.z), "=f"(t.w)
                 : "r"(a + 16 * m));
    v[2 * m] = make_float2(t.x, t.y);
    v[2 * m + 1] = make_float2(t.z, t.w);
  }
}

// Streamed loads: codes and scales through L2 only (each byte is read once
// per launch), v through the read-only path (the lanes of a row share it).
__device__ __forceinline__ void ld_cg_v4(uint32_t (&w)[4], const void* p) {
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
               : "l"(p));
}
__device__ __forceinline__ void ld_cg_v8(uint32_t (&w)[8], const void* p) {
  asm volatile("ld.global.cg.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
               : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]),
                 "=r"(w[7])
               : "l"(p));
}
__device__ __forceinline__ float ld_cg_f32(const float* p) {
  float x;
  asm volatile("ld.global.cg.f32 %0, [%1];\n" : "=f"(x) : "l"(p));
  return x;
}
__device__ __forceinline__ float ld_nc_f32(const float* p) {
  float x;
  asm volatile("ld.global.nc.f32 %0, [%1];\n" : "=f"(x) : "l"(p));
  return x;
}
__device__ __forceinline__ void st_global_v4(void* p, const uint32_t (&w)[4]) {
  asm volatile("st.global.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]),
               "r"(w[3])
               : "memory");
}

// One row block's streamed inputs of one lane.
template <int BITS>
struct BlockIn {
  uint32_t w[BITS];  // the lane's codes: BITS 32-bit words = 32 columns
  float s;           // the scale of the lane's group
  float v;           // v_i of the lane's row
};

template <int BITS>
__device__ __forceinline__ void load_block(BlockIn<BITS>& in, const uint8_t* codes, const float* scale,
                                           const float* v) {
  if constexpr (BITS == 4) {
    ld_cg_v4(in.w, codes);
  } else {
    ld_cg_v8(in.w, codes);
  }
  in.s = ld_cg_f32(scale);
  in.v = ld_nc_f32(v);
}

// (a & b) | c in one logic operation.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// INT4 chunk (4 two's complement words, column 8q + i at nibble i of word
// q) to the exact code values as pairs (2m, 2m+1).  After flipping every
// nibble's top bit (two's complement c becomes c + 8), nibble p of a 16-bit
// half of the word, kept in place at bit 4p and merged into e = the bits of
// 2^23, is the float 2^23 + 16^p (c + 8); one packed fused multiply-add per
// pair scales it by 16^-p and removes 2^23 16^-p + 8.  Both steps are exact.
__device__ __forceinline__ void unpack4(const uint32_t (&w)[4], float2 (&cv)[16], uint32_t e) {
  const float2 r01 = make_float2(1.0f, 0x1p-4f), r23 = make_float2(0x1p-8f, 0x1p-12f);
  const float2 b01 = make_float2(-(0x1p23f + 8.0f), -(0x1p19f + 8.0f));
  const float2 b23 = make_float2(-(0x1p15f + 8.0f), -(0x1p11f + 8.0f));
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t lo = w[q] ^ 0x88888888u, hi = lo >> 16;
    cv[4 * q + 0] = __ffma2_rn(make_float2(__uint_as_float(and_or(lo, 0xFu, e)),
                                           __uint_as_float(and_or(lo, 0xF0u, e))),
                               r01, b01);
    cv[4 * q + 1] = __ffma2_rn(make_float2(__uint_as_float(and_or(lo, 0xF00u, e)),
                                           __uint_as_float(and_or(lo, 0xF000u, e))),
                               r23, b23);
    cv[4 * q + 2] = __ffma2_rn(make_float2(__uint_as_float(and_or(hi, 0xFu, e)),
                                           __uint_as_float(and_or(hi, 0xF0u, e))),
                               r01, b01);
    cv[4 * q + 3] = __ffma2_rn(make_float2(__uint_as_float(and_or(hi, 0xF00u, e)),
                                           __uint_as_float(and_or(hi, 0xF000u, e))),
                               r23, b23);
  }
}

// A chunk's codes (BITS two's complement words) to exact values.
template <int BITS>
__device__ __forceinline__ void unpack_codes(const uint32_t (&w)[BITS], float2 (&cv)[16], uint32_t e) {
  if constexpr (BITS == 4) {
    unpack4(w, cv, e);
  } else {
    decode_chunk<8>(w, cv);
  }
}

// Pack 32 rounded values (floats kMagic + 2^(BITS-1) + n with n in
// [-qmax, qmax], as pairs (2m, 2m+1)) into BITS words of offset-binary
// fields n + 2^(BITS-1) (every field in [1, 2^BITS - 1]).
template <int BITS>
__device__ __forceinline__ void pack_offset(const float2 (&y)[16], uint32_t (&w)[BITS]) {
  if constexpr (BITS == 4) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t by[4];
#pragma unroll
      for (int b = 0; b < 4; ++b)
        by[b] = (__float_as_uint(y[4 * q + b].y) << 4) + __float_as_uint(y[4 * q + b].x);
      w[q] = __byte_perm(__byte_perm(by[0], by[1], 0x0040u), __byte_perm(by[2], by[3], 0x0040u), 0x5410u);
    }
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint32_t t0 = __byte_perm(__float_as_uint(y[2 * q].x), __float_as_uint(y[2 * q].y), 0x0040u);
      const uint32_t t1 =
          __byte_perm(__float_as_uint(y[2 * q + 1].x), __float_as_uint(y[2 * q + 1].y), 0x0040u);
      w[q] = __byte_perm(t0, t1, 0x5410u);
    }
  }
}

// Pack 32 rounded INT8 values (floats kMagic + 128 + n, as pairs
// (2m, 2m+1)) into 8 words of two's complement codes, saturating them to
// [-128, 127] on the way (the upper bound is qmax; the caller clamps the
// lower side to -qmax beforehand): cvt.pack.sat converts two 32-bit
// integers with saturation to the field's range and shifts them in below
// the word built so far (d = c << 16 | sat(a) << 8 | sat(b)).  The integer
// n is the float's bits less those of kMagic + 128: exact while the float
// lies in [2^23, 2^24); every larger float (huge or +infinite products)
// gives a larger integer, which saturates to qmax as the definition's clamp
// does.
__device__ __forceinline__ void pack_sat8(const float2 (&y)[16], uint32_t (&w)[8]) {
  constexpr float kOff = kMagic + 128.0f;
  const int off = static_cast<int>(__float_as_uint(kOff));
  auto n = [&](float v) { return static_cast<int>(__float_as_uint(v)) - off; };
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    // columns 4q .. 4q+3 = pairs 2q, 2q+1; the last pair goes in first
    uint32_t d = 0;
#pragma unroll
    for (int m = 1; m >= 0; --m)
      asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;"
          : "=r"(d)
          : "r"(n(y[2 * q + m].y)), "r"(n(y[2 * q + m].x)), "r"(d));
    w[q] = d;
  }
}

// Offset-binary INT4 words whose fields lie in [0, 15]; the codes' range
// is [1, 15] (code -7 .. 7), so every field equal to 0 steps up by one.  A
// field is nonzero when its top bit is set or adding 7 to its three low
// bits carries into the top bit.
__device__ __forceinline__ uint32_t int4_raise_zero(uint32_t w) {
  const uint32_t nonzero = ((w & 0x77777777u) + 0x77777777u) | w;
  return w + ((~nonzero & 0x88888888u) >> 3);
}

// Pack 32 rounded INT4 values (floats y = kMagic + 8 + n, as pairs
// (2m, 2m+1)) into 4 offset-binary words, fields m = n + 8 saturated to
// [0, 15].  One packed fused multiply-add takes y to (y - kMagic) 2^-149:
// y 2^-149 lies in [2^-126, 2^-125), where the float grid is 2^-149, so
// product and difference are exact and the result is m 2^-149, whose bits
// read as an integer are m itself (a subnormal for 0 <= m < 2^23).
// Smaller y (huge negative or -infinite products) give negative floats,
// whose bits read as a negative integer; larger y (huge or +infinite) give
// positive floats whose bits exceed 15.  cvt.pack.sat then saturates each
// to [0, 15] as the definition's clamp does (the caller raises 0 to 1) and
// shifts it in below the word built so far.
__device__ __forceinline__ void pack4_subnormal(const float2 (&y)[16], uint32_t (&w)[4]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t d = 0;
#pragma unroll
    for (int m = 3; m >= 0; --m) {
      const float2 z = __ffma2_rn(y[4 * q + m], f2(0x1p-149f), f2(-0x1.8p-126f));
      asm("cvt.pack.sat.u4.s32.b32 %0, %1, %2, %3;"
          : "=r"(d)
          : "r"(__float_as_uint(z.y)), "r"(__float_as_uint(z.x)), "r"(d));
    }
    w[q] = d;
  }
}

// The top bit of every field of a packed word (4-bit fields for INT4, 8-bit
// for INT8).
template <int BITS>
__host__ __device__ constexpr uint32_t field_tops() { return BITS == 4 ? 0x88888888u : 0x80808080u; }

// Bounded Directional Rounding under a fixed scale, on packed words.  With
// s' = s (persistent) and s a normal float, n s' < c s exactly when n < c,
// so the rule of include/qstate.h becomes an integer comparison of the new
// and the stored code, field by field.  N, C: offset-binary fields (code +
// 2^(BITS-1), new and stored, each in [1, 2^BITS - 1]); PF: every bit of
// the fields whose update sign sigma is > 0; AM: the lowest bit of the
// fields whose sigma is not 0, and of none where the rule is off for the
// word.  One comparison serves both directions: a field compares A = n,
// B = c where sigma > 0 and A = c, B = n where sigma < 0, and acts where
// A < B.  Unsigned x >= y per field: the borrow-free difference
// (x | top) - (y & ~top) compares the low bits, and its top bit combined
// with the fields' own top bits gives the full comparison.  The step of +-1
// moves a field toward c, so no carry or borrow crosses a field.
template <int BITS>
__device__ __forceinline__ uint32_t bdr_fixed_scale(uint32_t N, uint32_t C, uint32_t PF, uint32_t AM) {
  constexpr uint32_t H = field_tops<BITS>();
  const uint32_t A = (N & PF) | (C & ~PF);
  const uint32_t B = (C & PF) | (N & ~PF);
  const uint32_t z = (A | H) - (B & ~H);
  const uint32_t ge = (A & ~B) | (~(A ^ B) & z);  // top bits: A >= B
  const uint32_t act = ~(ge >> (BITS - 1)) & AM;  // lowest bits: A < B
  const uint32_t up = act & PF;
  return N + up - (act ^ up);
}

// Update-sign masks of a tile for the packed-word BDR, for this lane's 32
// columns: kpf / knf hold every bit of the fields whose key entry is > 0 /
// < 0, am the lowest bit of the fields whose key entry is not 0.
template <int BITS>
__device__ __forceinline__ void key_sign_masks(const float2 (&kk)[16], uint32_t (&kpf)[BITS],
                                               uint32_t (&knf)[BITS], uint32_t (&am)[BITS]) {
  constexpr int PER = 32 / BITS;  // fields per word
  constexpr uint32_t FIELD = (1u << BITS) - 1u;
#pragma unroll
  for (int q = 0; q < BITS; ++q) {
    uint32_t p = 0, n = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int j = q * PER + i;
      const float kv = (j & 1) ? kk[j >> 1].y : kk[j >> 1].x;
      const uint32_t f = FIELD << (BITS * i);
      p |= kv > 0.0f ? f : 0u;
      n |= kv < 0.0f ? f : 0u;
    }
    kpf[q] = p;
    knf[q] = n;
    am[q] = (p | n) & (field_tops<BITS>() >> (BITS - 1));
  }
}

// POLICY: 0 dynamic, 1 persistent.
template <int BITS, int DK, int POLICY, bool BDR, bool DELTA, bool DIAG>
__global__ void __maxnreg__(BDR ? (BITS == 8 ? QS_STREAM_REGS_BDR8 : QS_STREAM_REGS_BDR) : QS_STREAM_REGS)
    stream_step_kernel(StreamParams p) {
  static_assert(POLICY == 0 || POLICY == 1, "the yoked policy has its own kernel");
  constexpr int LPR = DK / 32;
  constexpr int RW = 32 / LPR;
  constexpr int CW = BITS;      // 32-bit code words per lane
  constexpr int CB = 4 * BITS;  // code bytes per lane
  constexpr int QMAX = BITS == 4 ? 7 : 127;
  constexpr float kQf = static_cast<float>(QMAX);
  constexpr float kOff = kMagic + (BITS == 4 ? 8.0f : 128.0f);
  constexpr unsigned CSTRIDE = RW * DK * BITS / 8;  // code bytes per row block
  constexpr uint32_t TOPS = field_tops<BITS>();
  // the packed-word form of BDR needs the fixed scale
  constexpr bool BDR_WORDS = BDR && POLICY == 1;
  constexpr bool BDR_FLOAT = BDR && POLICY == 0;
  // fixed scales the packed-word BDR and the fast reciprocal take directly
  constexpr float kScaleHi = POLICY == 1 ? 0x1p100f : 0x1p126f;
  constexpr bool KS = QS_STREAM_K_SMEM < 0 ? BDR : QS_STREAM_K_SMEM != 0;

  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31;
  const int c = lane % LPR, rr = lane / LPR;
  const StreamLayout L(DK, DIAG, BDR_FLOAT);
  const unsigned ng = DK / p.group;
  const unsigned g = (32 * c) / p.group;
  const bool readout = p.o != nullptr;
  const bool writes_scale = (32 * c) % p.group == 0;
  const uint32_t e23 = p.two23;

  // this warp's contiguous range of row blocks
  const long long nw = static_cast<long long>(gridDim.x);
  const unsigned b0 = static_cast<unsigned>(blockIdx.x * static_cast<long long>(p.nblocks) / nw);
  const unsigned b1 = static_cast<unsigned>((blockIdx.x + 1) * static_cast<long long>(p.nblocks) / nw);
  if (b0 >= b1) return;
  const unsigned bpt = static_cast<unsigned>(p.bpt);

  // per-lane bases; row block b adds b times a per-block stride (one wide
  // multiply-add of the 32-bit block index per address)
  const unsigned sstride = RW * ng;
  uint8_t* const codes_l = p.codes + CB * lane;
  float* const scales_l = p.scales + rr * ng + g;
  const float* const v_l = p.v + rr;
  float* const o_l = p.o + rr;
  auto codes_at = [&](unsigned b) { return codes_l + static_cast<unsigned long long>(b) * CSTRIDE; };
  auto scale_at = [&](unsigned b) { return scales_l + static_cast<unsigned long long>(b) * sstride; };
  auto v_at = [&](unsigned b) { return v_l + static_cast<unsigned long long>(b) * RW; };

  // INT4: the first two row blocks' codes and scales toward L2 while the
  // previous kernel of the stream finishes (the INT8 instances, at their
  // register cap, would spill for it)
  if constexpr (BITS == 4) {
    prefetch_l2(codes_at(b0));
    prefetch_l2(scale_at(b0));
    if (b0 + 1 < b1) {
      prefetch_l2(codes_at(b0 + 1));
      prefetch_l2(scale_at(b0 + 1));
    }
  }
  grid_dep_wait();
  grid_dep_launch();

  // ---- per-tile vectors: cp.async into the warp's two slots
  const uint32_t slots = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  auto stage_tile = [&](unsigned t, int slot) {
    const uint32_t base = slots + slot * L.slot;
    if (lane < DK / 4) {
      const uint32_t u = base + static_cast<uint32_t>(vec_unit_offset(lane));
      const size_t off = static_cast<size_t>(t) * DK + 4 * lane;
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(u + L.k), "l"(p.k + off) : "memory");
      if (readout)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(u + L.q), "l"(p.q + off) : "memory");
      if constexpr (DIAG)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(u + L.a), "l"(p.alpha + off)
                     : "memory");
    }
    if (lane == 0 && !DIAG)
      asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(base + L.misc), "l"(p.alpha + t)
                   : "memory");
    if (lane == 1)
      asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(base + L.misc + 4), "l"(p.beta + t)
                   : "memory");
  };

  unsigned tile = b0 / bpt;
  unsigned tile_end = (tile + 1) * bpt;  // first row block of the next tile
  int slot = 0;
  stage_tile(tile, 0);
  cp_async_commit();
  if (tile_end < b1) stage_tile(tile + 1, 1);
  cp_async_commit();

  BlockIn<BITS> A, B;
  load_block<BITS>(A, codes_at(b0), scale_at(b0), v_at(b0));
  if (b0 + 1 < b1) load_block<BITS>(B, codes_at(b0 + 1), scale_at(b0 + 1), v_at(b0 + 1));

  float2 kk[16];
  float beta = 0.0f, a_scalar = 1.0f;
  uint32_t kp[BDR_WORDS ? CW : 1], kn[BDR_WORDS ? CW : 1], am[BDR_WORDS ? CW : 1];
  const unsigned char* tv = smem;
  auto enter_tile = [&]() {
    tv = smem + slot * L.slot;
    if constexpr (KS) {
      if constexpr (BDR) load_pairs(tv + L.k, c, kk);   // for the sign masks only
    } else {
      load_pairs(tv + L.k, c, kk);
    }
    const float* misc = reinterpret_cast<const float*>(tv + L.misc);
    beta = misc[1];
    a_scalar = DIAG ? 1.0f : misc[0];
    if constexpr (BDR_WORDS) key_sign_masks<BITS>(kk, kp, kn, am);
    if constexpr (BDR_FLOAT) {
      // sign(k_j) per column, in the layout of k, written once per tile
      if (rr == 0) {
        float* ss = reinterpret_cast<float*>(const_cast<unsigned char*>(tv) + L.sk) + c * kChunkStride;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          ss[2 * m] = kk[m].x > 0.0f ? 1.0f : (kk[m].x < 0.0f ? -1.0f : 0.0f);
          ss[2 * m + 1] = kk[m].y > 0.0f ? 1.0f : (kk[m].y < 0.0f ? -1.0f : 0.0f);
        }
      }
      __syncwarp();
    }
  };
  cp_async_wait<1>();
  __syncwarp();
  enter_tile();

  // One row block: the whole step for this lane's 32 elements.  `in` is
  // refilled with row block b + 2 as soon as its codes are unpacked.
  auto row_block = [&](BlockIn<BITS>& in, unsigned b) {
    // ---- a1: unpack
    float2 Sp[16];
    unpack_codes<BITS>(in.w, Sp, e23);
    uint32_t cold[BDR_WORDS ? CW : 1];
    if constexpr (BDR_WORDS) {
#pragma unroll
      for (int q = 0; q < CW; ++q) cold[q] = in.w[q] ^ TOPS;  // offset binary
    }
    const float s_old = in.s, v_i = in.v;
    // BDR's reference under a changing scale: d = c * s
    float2 dref[BDR_FLOAT ? 16 : 1];
    if constexpr (BDR_FLOAT) {
#pragma unroll
      for (int m = 0; m < 16; ++m) dref[m] = __fmul2_rn(Sp[m], f2(s_old));
    }
    if (b + 2 < b1) load_block<BITS>(in, codes_at(b + 2), scale_at(b + 2), v_at(b + 2));

    // ---- a2: dequantize with the decayed scale, S' = c * (s * a)
    if constexpr (DIAG) {
      float2 aa[16];
      load_pairs(tv + L.a, c, aa);
#pragma unroll
      for (int m = 0; m < 16; ++m) Sp[m] = __fmul2_rn(Sp[m], __fmul2_rn(f2(s_old), aa[m]));
    } else {
      const float sa = __fmul_rn(s_old, a_scalar);
#pragma unroll
      for (int m = 0; m < 16; ++m) Sp[m] = __fmul2_rn(Sp[m], f2(sa));
    }

    // ---- a3/a4: key projection and rank-1 write
    float wcoef;
    if constexpr (DELTA) {
      float2 ku[16];
      if constexpr (KS) load_pairs_v(tv + L.k, c, ku);
      const float2(&k1)[16] = KS ? ku : kk;
      wcoef = __fmul_rn(beta, __fsub_rn(v_i, row_tree<LPR>(chunk_sum(Sp, k1))));
    } else {
      wcoef = __fmul_rn(beta, v_i);
    }
    float2 x[16];
    {
      float2 kx[16];
      if constexpr (KS) load_pairs_v(tv + L.k, c, kx);
      const float2(&k2)[16] = KS ? kx : kk;
#pragma unroll
      for (int m = 0; m < 16; ++m) x[m] = __ffma2_rn(f2(wcoef), k2[m], Sp[m]);
    }

    // ---- a5: readout from the updated state
    if (readout) {
      ChunkDot acc;
      const float4* qp4 = reinterpret_cast<const float4*>(tv + L.q) + c * (kChunkStride / 4);
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const float4 t = qp4[m];
        acc.add(2 * m, x[2 * m], make_float2(t.x, t.y));
        acc.add(2 * m + 1, x[2 * m + 1], make_float2(t.z, t.w));
      }
      const float o = row_tree<LPR>(acc.sum());
      if (c == 0) o_l[static_cast<unsigned long long>(b) * RW] = o;
    }

    // ---- a7: scale; a8: round (persistent scales clamp every element: huge,
    // infinite and NaN products included, they land outside the range and
    // clamp to the side the definition gives)
    float sp, inv, m = 0.0f;
    if constexpr (POLICY == 0) {
      m = row_max<LPR>(chunk_absmax(x), p.group);
      sp = div_qmax_fast<QMAX>(m);
    } else {
      sp = s_old;
    }
    inv = recip_fast(sp);
    bool normal = sp >= 0x1p-126f && sp < kScaleHi;
    if constexpr (POLICY == 0) normal = normal && m <= 3.40282347e38f;
    float2 y[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) y[i] = __ffma2_rn(x[i], f2(inv), f2(kOff));
    if constexpr (POLICY == 1 && BITS == 8) {
      // the lower side of the clamp; pack_sat8 clamps the upper side (INT4
      // raises -8 to -7 on the packed words instead)
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        y[i].x = fmaxf(y[i].x, kOff - kQf);
        y[i].y = fmaxf(y[i].y, kOff - kQf);
      }
    }
    // The fast forms above are exact for a finite group max and a scale in
    // [2^-126, kScaleHi).  Any other scale (zero, subnormal, huge, infinite,
    // NaN) takes the general routines in a branch the whole warp enters.
    bool zero = false;
    uint32_t words_on = ~0u;  // packed-word BDR allowed for this lane
    if (__any_sync(0xffffffffu, !normal)) {
      if (!normal) {
        if constexpr (POLICY == 0) sp = div_qmax_rn<QMAX>(m);
        zero = !(sp > 0.0f);
        inv = zero ? 0.0f : recip_rn(sp);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 t = __ffma2_rn(x[i], f2(inv), f2(kOff));
          y[i].x = zero ? kOff : fminf(fmaxf(t.x, kOff - kQf), kOff + kQf);
          y[i].y = zero ? kOff : fminf(fmaxf(t.y, kOff - kQf), kOff + kQf);
        }
        if constexpr (BDR_WORDS) {
          // a subnormal fixed scale keeps products of distinct codes distinct,
          // so the packed words still decide; a scale of 2^100 or more may
          // overflow n s', so those lanes take the dequantized comparison
          words_on = 0u;
          if (!zero && sp < kScaleHi) words_on = ~0u;
          const float swf = wcoef > 0.0f ? 1.0f : (wcoef < 0.0f ? -1.0f : 0.0f);
          if (!zero && !(sp < kScaleHi)) {
            uint32_t wold[CW];
#pragma unroll
            for (int q = 0; q < CW; ++q) wold[q] = cold[q] ^ TOPS;
            float2 cv[16], dd[16], sk[16], kr[16];
            load_pairs_v(tv + L.k, c, kr);
            unpack_codes<BITS>(wold, cv, e23);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              dd[i] = __fmul2_rn(cv[i], f2(s_old));
              sk[i] = make_float2(kr[i].x > 0.0f ? 1.0f : (kr[i].x < 0.0f ? -1.0f : 0.0f),
                                  kr[i].y > 0.0f ? 1.0f : (kr[i].y < 0.0f ? -1.0f : 0.0f));
            }
            bdr_chunk<BITS>(y, dd, sk, swf, sp);
          }
        }
      }
    }
    if constexpr (BDR_FLOAT) {
      const float sw = zero ? 0.0f : (wcoef > 0.0f ? 1.0f : (wcoef < 0.0f ? -1.0f : 0.0f));
      float2 sk[16];
      load_pairs(tv + L.sk, c, sk);
      bdr_chunk<BITS>(y, dref, sk, sw, sp);
    }

    // ---- a9: pack (and BDR on the packed words), store
    uint32_t out[CW];
    if constexpr (POLICY == 1) {
      // offset-binary words from a saturating pack, compared with the stored
      // words in offset binary, then flipped back to two's complement
      if constexpr (BITS == 4) {
        pack4_subnormal(y, out);
#pragma unroll
        for (int q = 0; q < CW; ++q) out[q] = int4_raise_zero(out[q]);
      } else {
        pack_sat8(y, out);
#pragma unroll
        for (int q = 0; q < CW; ++q) out[q] ^= TOPS;
      }
      if constexpr (BDR_WORDS) {
        const bool pos = wcoef > 0.0f;
        const uint32_t on = (wcoef != 0.0f) ? words_on : 0u;
#pragma unroll
        for (int q = 0; q < CW; ++q) {
          out[q] = bdr_fixed_scale<BITS>(out[q], cold[q], pos ? kp[q] : kn[q], am[q] & on);
        }
      }
#pragma unroll
      for (int q = 0; q < CW; ++q) out[q] ^= TOPS;
    } else {
      pack_offset<BITS>(y, out);
#pragma unroll
      for (int q = 0; q < CW; ++q) out[q] ^= TOPS;
    }
    if constexpr (CW == 4) {
      st_global_v4(codes_at(b), out);
    } else {
      st_global_v8(codes_at(b), out);
    }
    if constexpr (POLICY == 0) {
      if (writes_scale) *scale_at(b) = sp;
    }
  };

  // alternate the two register sets; switch tiles between row blocks
  auto next = [&](unsigned b) {
    if (b == tile_end) {
      ++tile;
      tile_end += bpt;
      slot ^= 1;
      cp_async_wait<0>();
      // every lane's copies of this tile have landed, and every lane is done
      // with the slot that the next tile's copies overwrite
      __syncwarp();
      enter_tile();
      if (tile_end < b1) stage_tile(tile + 1, slot ^ 1);
      cp_async_commit();
    }
  };
  unsigned b = b0;
#pragma unroll 1
  while (true) {
    row_block(A, b);
    if (++b >= b1) break;
    next(b);
    row_block(B, b);
    if (++b >= b1) break;
    next(b);
  }
  cp_async_wait<0>();
}

}  // namespace qs
