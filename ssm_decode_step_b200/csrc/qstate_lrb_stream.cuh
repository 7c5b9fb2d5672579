// Low-Rank Bypass, the steps that leave the stored state as it is (sm_100a):
// the streamed form of qstate_lrb_decode_step for every slot of a period but
// the last, under the dynamic and persistent policies ("Preserving Updates in
// Low-Bit Recurrent State Quantization", abstract: small updates accumulate
// in a compact low-rank buffer and are merged into the state periodically).
//
// Such a step reads the codes and scales and writes no code: per row
//   S'_j  = c_j (s A_j)                       (A = A_in a, the accumulated decay)
//   u     = S'.k + sum_r U_r (K'_r . k)       (delta rule only)
//   w     = beta (v - u)       or  beta v
//   o     = S'.q + sum_r U_r (K'_r . q) + w (k . q)
//   U_slot = w
// with K'_r = K_in_r a the buffered keys decayed by this step, in the fixed
// operation order of include/qstate.h.  The work decomposition is the plain
// streamed step's (qstate_stream.cuh): one warp per CTA, a contiguous range of
// row blocks per warp, each lane's codes, scale, v and its row's buffered
// coefficients U loaded into registers two row blocks ahead, and each tile's
// vectors (k, q, the step's decay, A_in and the buffered keys) staged by
// cp.async into one of two shared-memory slots a tile ahead.  On entering a
// tile a warp forms A, the decayed keys and their products with k and q; the
// warp whose range holds the tile's first row block also writes A_out and
// K_out (the caller swaps the two copies between steps, so no warp reads what
// another writes in the launch).  Per row block each code word is unpacked,
// dequantized and fed to both dot products' chains at once.  The last slot of
// a period (the merge) and every slot of the yoked policy run the ring kernel
// of qstate_lrb.cuh.
#pragma once

#include "qstate_lrb.cuh"
#include "qstate_stream.cuh"

// Registers per thread of the bypass kernel: 168 leave 12 resident warps per
// SM for INT4 with ranks up to 8; INT8 and ranks up to 16 (twice the code
// words or coefficient units in flight) get 200 (10 warps).
#ifndef QS_BYPASS_REGS
#define QS_BYPASS_REGS 168
#endif
#ifndef QS_BYPASS_REGS8
#define QS_BYPASS_REGS8 200
#endif

namespace qs {

// One warp's shared memory: two tile slots, each holding k, q, the step's
// diagonal decay, A_in and up to `rows` buffered keys at the padded chunk
// stride, then the products K'_r . k and K'_r . q, then alpha and beta.
struct BypassLayout {
  int k, q, a, A, Kb, kdot, qdot, misc, slot;
  __host__ __device__ BypassLayout(int dk, bool diag, int rows) {
    const int vec = (dk / 32) * kChunkStride * 4;
    int off = 0;
    k = off;    off += vec;
    q = off;    off += vec;
    a = off;    off += diag ? vec : 0;
    A = off;    off += vec;
    Kb = off;   off += rows * vec;
    kdot = off; off += kLrbMaxRank * 4;
    qdot = off; off += kLrbMaxRank * 4;
    misc = off; off += 16;
    slot = align_up(off, 128);
  }
  __host__ __device__ int bytes() const { return 2 * slot; }
};

// One row block's streamed inputs of one lane: codes, scale, v and its
// row's buffered coefficients U_r in 16-byte units (MAXU units: the period's
// rank rounded up to 4, at most 8 or 16; only the (slot + 3) / 4 units that
// hold buffered terms are loaded).
template <int BITS, int MAXU>
struct BypassIn {
  uint32_t w[BITS];
  float s;
  float v;
  float4 u[MAXU];
};

__device__ __forceinline__ float4 ld_cg_f4(const float* p) {
  float4 x;
  asm volatile("ld.global.cg.v4.f32 {%0,%1,%2,%3}, [%4];\n"
               : "=f"(x.x), "=f"(x.y), "=f"(x.z), "=f"(x.w)
               : "l"(p));
  return x;
}

// A chunk a against chunk c of a staged Dk vector read from shared memory as
// it is used (volatile: no copy of the vector stays in registers), in the
// fixed order of chunk_sum.
__device__ __forceinline__ float chunk_sum_sv(const float2 (&a)[16], const unsigned char* base, int c) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(base)) + c * (kChunkStride * 4);
  ChunkDot d;
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    float4 t;
    asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];\n"
                 : "=f"(t.x), "=f"(t.y), "=f"(t.z), "=f"(t.w)
                 : "r"(s + 16 * m));
    d.add(2 * m, a[2 * m], make_float2(t.x, t.y));
    d.add(2 * m + 1, a[2 * m + 1], make_float2(t.z, t.w));
  }
  return d.sum();
}

// Code word q of a lane's chunk to its exact code values, as the pairs of
// columns it holds: INT4 word q holds columns 8q .. 8q+7 (pairs 4q .. 4q+3;
// the steps of unpack4), INT8 word q columns 4q .. 4q+3 (pairs 2q, 2q+1; the
// steps of decode_chunk).
template <int BITS>
__device__ __forceinline__ void unpack_word(uint32_t w, float2 (&cv)[BITS == 4 ? 4 : 2], uint32_t e) {
  if constexpr (BITS == 4) {
    const uint32_t lo = w ^ 0x88888888u, hi = lo >> 16;
    const float2 r01 = make_float2(1.0f, 0x1p-4f), r23 = make_float2(0x1p-8f, 0x1p-12f);
    const float2 b01 = make_float2(-(0x1p23f + 8.0f), -(0x1p19f + 8.0f));
    const float2 b23 = make_float2(-(0x1p15f + 8.0f), -(0x1p11f + 8.0f));
    cv[0] = __ffma2_rn(make_float2(__uint_as_float(and_or(lo, 0xFu, e)), __uint_as_float(and_or(lo, 0xF0u, e))),
                       r01, b01);
    cv[1] = __ffma2_rn(make_float2(__uint_as_float(and_or(lo, 0xF00u, e)), __uint_as_float(and_or(lo, 0xF000u, e))),
                       r23, b23);
    cv[2] = __ffma2_rn(make_float2(__uint_as_float(and_or(hi, 0xFu, e)), __uint_as_float(and_or(hi, 0xF0u, e))),
                       r01, b01);
    cv[3] = __ffma2_rn(make_float2(__uint_as_float(and_or(hi, 0xF00u, e)), __uint_as_float(and_or(hi, 0xF000u, e))),
                       r23, b23);
  } else {
    const uint32_t x = w ^ 0x80808080u;
#pragma unroll
    for (int h = 0; h < 2; ++h)
      cv[h] = __fadd2_rn(make_float2(__uint_as_float(__byte_perm(x, 0x4B000000u, 0x7540u | (2 * h))),
                                     __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7540u | (2 * h + 1)))),
                         f2(-8388736.0f));
  }
}

template <int BITS, int DK, bool DELTA, bool DIAG, int MAXU>
__global__ void __maxnreg__((BITS == 8 || MAXU > 2) ? QS_BYPASS_REGS8 : QS_BYPASS_REGS)
    lrb_bypass_kernel(LrbParams p) {
  constexpr int LPR = DK / 32;
  constexpr int RW = 32 / LPR;
  constexpr int CB = 4 * BITS;  // code bytes per lane
  constexpr unsigned CSTRIDE = RW * DK * BITS / 8;
  constexpr int VU = DK / 4;    // 16-byte units of a Dk vector
  constexpr int VEC = LPR * kChunkStride * 4;

  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x;
  const int c = lane % LPR, rr = lane / LPR;
  const BypassLayout L(DK, DIAG, p.rank);
  const unsigned ng = DK / p.group;
  const unsigned g = (32 * c) / p.group;
  const bool readout = p.o != nullptr;
  const int nbuf = p.slot;  // buffered terms: the period's earlier steps
  const int units = (nbuf + 3) >> 2;
  const uint32_t e23 = p.two23;

  // this warp's contiguous range of row blocks
  const long long nw = static_cast<long long>(gridDim.x);
  const unsigned b0 = static_cast<unsigned>(blockIdx.x * static_cast<long long>(p.nblocks) / nw);
  const unsigned b1 = static_cast<unsigned>((blockIdx.x + 1) * static_cast<long long>(p.nblocks) / nw);
  if (b0 >= b1) return;
  const unsigned bpt = static_cast<unsigned>(p.bpt);
  grid_dep_wait();
  grid_dep_launch();

  const unsigned sstride = RW * ng;
  const unsigned ustride = RW * p.rpad;
  const uint8_t* const codes_l = p.codes + CB * lane;
  const float* const scales_l = p.scales + rr * ng + g;
  const float* const v_l = p.v + rr;
  float* const o_l = p.o + rr;
  float* const u_l = p.U + rr * p.rpad;
  auto load = [&](BypassIn<BITS, MAXU>& in, unsigned b) {
    const uint8_t* cp = codes_l + static_cast<unsigned long long>(b) * CSTRIDE;
    if constexpr (BITS == 4) {
      ld_cg_v4(in.w, cp);
    } else {
      ld_cg_v8(in.w, cp);
    }
    in.s = ld_cg_f32(scales_l + static_cast<unsigned long long>(b) * sstride);
    in.v = ld_nc_f32(v_l + static_cast<unsigned long long>(b) * RW);
    const float* ur = u_l + static_cast<unsigned long long>(b) * ustride;
#pragma unroll
    for (int i = 0; i < MAXU; ++i)
      if (i < units) in.u[i] = ld_cg_f4(ur + 4 * i);
  };

  // ---- per-tile vectors: cp.async into the warp's two slots
  const uint32_t slots = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  auto stage_tile = [&](unsigned t, int sl) {
    const uint32_t base = slots + sl * L.slot;
    if (lane < VU) {
      const uint32_t u = base + static_cast<uint32_t>(vec_unit_offset(lane));
      const size_t off = static_cast<size_t>(t) * DK + 4 * lane;
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(u + L.k), "l"(p.k + off) : "memory");
      if (readout)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(u + L.q), "l"(p.q + off) : "memory");
      if constexpr (DIAG)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(u + L.a), "l"(p.alpha + off)
                     : "memory");
      if (nbuf > 0)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(u + L.A), "l"(p.A_in + off)
                     : "memory");
    }
    // the buffered keys K_in_r, r < slot
    const float* kin = p.K_in + static_cast<size_t>(t) * p.rank * DK;
    for (int i = lane; i < nbuf * VU; i += 32) {
      const int r = i / VU, u = i % VU;
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(base + L.Kb + r * VEC +
                                                                         vec_unit_offset(u)),
                   "l"(kin + r * DK + 4 * u)
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
  int sl = 0;
  stage_tile(tile, 0);
  cp_async_commit();
  if (tile_end < b1) stage_tile(tile + 1, 1);
  cp_async_commit();

  BypassIn<BITS, MAXU> X{}, Y{};  // coefficient units past the buffer stay 0
  load(X, b0);
  if (b0 + 1 < b1) load(Y, b0 + 1);

  // ---- entering a tile: A = A_in a, the decayed buffered keys and their
  // products with k and q, k . q; the tile's writer stores A_out and K_out
  float2 kk[16], qq[16];
#pragma unroll
  for (int m = 0; m < 16; ++m) kk[m] = qq[m] = make_float2(0.0f, 0.0f);
  float beta = 0.0f, a_acc = 1.0f, kqn = 0.0f;
  const unsigned char* tv = smem;
  auto enter_tile = [&](unsigned b) {
    tv = smem + sl * L.slot;
    const float* misc = reinterpret_cast<const float*>(tv + L.misc);
    beta = misc[1];
    const float a_step = DIAG ? 1.0f : misc[0];
    // this step's decay over the lane's chunk (diagonal: re-read from the
    // slot at each use, so that it holds no registers across the tile)
    auto decay = [&](float2 (&aa)[16]) {
      if constexpr (DIAG) {
        load_pairs_v(tv + L.a, c, aa);
      } else {
#pragma unroll
        for (int m = 0; m < 16; ++m) aa[m] = f2(a_step);
      }
    };
    float2 A[16];
    {
      float2 aa[16];
      decay(aa);
      if (nbuf == 0) {
#pragma unroll
        for (int m = 0; m < 16; ++m) A[m] = aa[m];
      } else {
        load_pairs(tv + L.A, c, A);
#pragma unroll
        for (int m = 0; m < 16; ++m) A[m] = __fmul2_rn(A[m], aa[m]);
      }
    }
    if constexpr (DIAG) {
      // A replaces A_in in the slot, read by every row block of the tile
      __syncwarp();
      if (rr == 0) {
        float* dA = reinterpret_cast<float*>(const_cast<unsigned char*>(tv) + L.A) + c * kChunkStride;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          dA[2 * m] = A[m].x;
          dA[2 * m + 1] = A[m].y;
        }
      }
    } else {
      a_acc = A[0].x;  // scalar decay: every A_j of the tile is the same product
    }
    const size_t t = tile;
    const bool writer = b == tile * bpt;
    if (writer && rr == 0) {
      float4* gA = reinterpret_cast<float4*>(p.A_out + t * DK + 32 * c);
#pragma unroll
      for (int m = 0; m < 8; ++m) gA[m] = make_float4(A[2 * m].x, A[2 * m].y, A[2 * m + 1].x, A[2 * m + 1].y);
    }
    // k and q stay in shared memory until the tile's products are formed,
    // so that the registers they take in the row blocks are free here
    {
      float2 kt[16];
      load_pairs_v(tv + L.k, c, kt);
      if (writer && rr == 0) {
        float4* gK = reinterpret_cast<float4*>(p.K_out + (t * p.rank + nbuf) * DK + 32 * c);
#pragma unroll
        for (int m = 0; m < 8; ++m) gK[m] = make_float4(kt[2 * m].x, kt[2 * m].y, kt[2 * m + 1].x, kt[2 * m + 1].y);
      }
      if (readout) kqn = row_tree<LPR>(chunk_sum_sv(kt, tv + L.q, c));
    }
    float* kdot = reinterpret_cast<float*>(const_cast<unsigned char*>(tv) + L.kdot);
    float* qdot = reinterpret_cast<float*>(const_cast<unsigned char*>(tv) + L.qdot);
    for (int r0 = 0; r0 < nbuf; r0 += RW) {
      // every lane takes part in the row reductions; rows past the buffer
      // reduce zeros and store nothing
      const int r = r0 + rr;
      const bool live = r < nbuf;
      float2 Kr[16], aa[16];
      load_pairs(tv + L.Kb + (live ? r : 0) * VEC, c, Kr);
      decay(aa);
#pragma unroll
      for (int m = 0; m < 16; ++m) Kr[m] = live ? __fmul2_rn(Kr[m], aa[m]) : make_float2(0.0f, 0.0f);
      float kd = 0.0f, qd = 0.0f;
      if constexpr (DELTA) kd = row_tree<LPR>(chunk_sum_sv(Kr, tv + L.k, c));
      if (readout) qd = row_tree<LPR>(chunk_sum_sv(Kr, tv + L.q, c));
      if (live) {
        if (c == 0) {
          kdot[r] = kd;
          qdot[r] = qd;
        }
        if (writer) {
          float4* gK = reinterpret_cast<float4*>(p.K_out + (t * p.rank + r) * DK + 32 * c);
#pragma unroll
          for (int m = 0; m < 8; ++m)
            gK[m] = make_float4(Kr[2 * m].x, Kr[2 * m].y, Kr[2 * m + 1].x, Kr[2 * m + 1].y);
        }
      }
    }
    __syncwarp();
    // k and q in registers for the row blocks of the tile
    if constexpr (DELTA) load_pairs(tv + L.k, c, kk);
    if (readout) load_pairs(tv + L.q, c, qq);
  };
  cp_async_wait<1>();
  __syncwarp();
  enter_tile(b0);

  // One row block: this lane's 32 columns of row b RW + rr.  `in` is
  // refilled with row block b + 2 once its values are used.
  auto row_block = [&](BypassIn<BITS, MAXU>& in, unsigned b) {
    const float s_old = in.s, v_i = in.v;
    // word by word: codes to values, S' = c (s A_j), and both dot products'
    // chains (pair m feeds chain m mod 4 of each, in the order of m)
    constexpr int PW = BITS == 4 ? 4 : 2;  // pairs per code word
    const float sa = DIAG ? 0.0f : __fmul_rn(s_old, a_acc);
    const float4* A4 = reinterpret_cast<const float4*>(tv + L.A) + c * (kChunkStride / 4);
    ChunkDot dk, dq;
#pragma unroll
    for (int q = 0; q < BITS; ++q) {
      float2 cv[PW];
      unpack_word<BITS>(in.w[q], cv, e23);
#pragma unroll
      for (int e = 0; e < PW; ++e) {
        const int m = q * PW + e;
        float2 sp;
        if constexpr (DIAG) {
          const float4 a4 = A4[m >> 1];
          const float2 a = (m & 1) ? make_float2(a4.z, a4.w) : make_float2(a4.x, a4.y);
          sp = __fmul2_rn(cv[e], __fmul2_rn(f2(s_old), a));
        } else {
          sp = __fmul2_rn(cv[e], f2(sa));
        }
        // (without a readout q is not staged and dq is not used)
        if constexpr (DELTA) dk.add(m, sp, kk[m]);
        dq.add(m, sp, qq[m]);
      }
    }
    // then the buffer's terms U_r (K'_r . k) and U_r (K'_r . q), r < slot,
    // continuing each chain in the order of r
    float ua = 0.0f;
    if constexpr (DELTA) ua = row_tree<LPR>(dk.sum());
    float oa = row_tree<LPR>(dq.sum());
    const float4* kd4 = reinterpret_cast<const float4*>(tv + L.kdot);
    const float4* qd4 = reinterpret_cast<const float4*>(tv + L.qdot);
#pragma unroll
    for (int i = 0; i < MAXU; ++i) {
      const float4 kd = kd4[i], qd = qd4[i];
      const float uv[4] = {in.u[i].x, in.u[i].y, in.u[i].z, in.u[i].w};
      const float kv[4] = {kd.x, kd.y, kd.z, kd.w};
      const float qv[4] = {qd.x, qd.y, qd.z, qd.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool live = 4 * i + e < nbuf;  // the same for every lane
        if constexpr (DELTA) ua = live ? __fmaf_rn(uv[e], kv[e], ua) : ua;
        oa = live ? __fmaf_rn(uv[e], qv[e], oa) : oa;
      }
    }
    if (b + 2 < b1) load(in, b + 2);
    // write coefficient against S' + sum_r U_r K'_r^T
    float wcoef;
    if constexpr (DELTA) {
      wcoef = __fmul_rn(beta, __fsub_rn(v_i, ua));
    } else {
      wcoef = __fmul_rn(beta, v_i);
    }
    if (readout) {
      const float o = __fmaf_rn(wcoef, kqn, oa);
      if (c == 0) o_l[static_cast<unsigned long long>(b) * RW] = o;
    }
    // the write joins the buffer; the stored state is kept
    if (c == 0) u_l[static_cast<unsigned long long>(b) * ustride + nbuf] = wcoef;
  };

  auto next = [&](unsigned b) {
    if (b == tile_end) {
      ++tile;
      tile_end += bpt;
      sl ^= 1;
      cp_async_wait<0>();
      // every lane's copies of this tile have landed, and every lane is done
      // with the slot that the next tile's copies overwrite
      __syncwarp();
      enter_tile(b);
      if (tile_end < b1) stage_tile(tile + 1, sl ^ 1);
      cp_async_commit();
    }
  };
  unsigned b = b0;
#pragma unroll 1
  while (true) {
    row_block(X, b);
    if (++b >= b1) break;
    next(b);
    row_block(Y, b);
    if (++b >= b1) break;
    next(b);
  }
  cp_async_wait<0>();
}

}  // namespace qs
