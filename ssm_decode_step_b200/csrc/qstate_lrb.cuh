// Low-Rank Bypass decode step (sm_100a): qstate_lrb_decode_step.
//
// The writes of a period of `rank` steps bypass the quantized state: they
// are held as FP32 rank-1 terms w k^T (coefficients U [T][Dv][rpad], keys
// K [T][rank][Dk] decayed in place), the stored codes are left as they are
// with their decay accumulated per column in A [T][Dk], and the last step of
// the period (MERGE) adds the buffer to the state and requantizes it once.
// The element-level definition and the fixed operation order are those of
// include/qstate.h (qstate_lrb_decode_step); the work decomposition, ring
// and tile-vector slots are those of the plain step (qstate_step.cuh).
//
// Per tile, at the first row block a warp computes of it: A = A_in * a,
// the decayed keys K'_r = K_in_r * a (r < slot), kk_r = K'_r . k,
// kq_r = K'_r . q and kqn = k . q, into the warp's tile-vector slot.  The
// warp whose range holds the tile's first row block also writes A_out,
// K_out (bypass steps only); every other warp only reads A_in and K_in, so
// no warp reads what another writes in the same launch.
#pragma once

#include "qstate_step.cuh"

namespace qs {

constexpr int kLrbMaxRank = 16;

struct LrbParams {
  uint8_t* codes;
  float* scales;
  float* shadow;
  const float* q;
  const float* k;
  const float* v;
  const float* alpha;
  const float* beta;
  float* o;
  const float* A_in;
  float* A_out;
  const float* K_in;
  float* K_out;
  float* U;        // [T][Dv][rpad]
  int nblocks;
  int bpt;
  int group;
  int ntv;
  int warp_bytes;
  int rank;
  int rpad;        // rank rounded up to a multiple of 4
  int slot;        // position of this step in the period
  uint32_t two23;  // the bits of 2^23 for the streamed INT4 unpack
};

// One warp's shared memory: DEPTH ring slots, then ntv tile-vector slots.
struct LrbLayout {
  int slot, codes, scales, v, u, shadow;        // ring slot
  int tv, k, q, a, A, Kb, kdot, qdot, misc;     // tile-vector slot
  __host__ __device__ LrbLayout(int bits, int dk, bool diag, bool yoked, bool merge, int rank,
                                int rpad) {
    const int rw = 32 / (dk / 32);
    int off = 0;
    codes = off;  off += 32 * 4 * bits;
    scales = off; off += 32 * 4;
    v = off;      off += 32 * 4;
    u = off;      off += rw * rpad * 4;
    shadow = off; off += yoked ? 32 * kShadowStride : 0;
    slot = align_up(off, 16);
    const int vec = (dk / 32) * kChunkStride * 4;
    off = 0;
    k = off;    off += vec;
    q = off;    off += vec;
    a = off;    off += diag ? vec : 0;
    A = off;    off += vec;
    Kb = off;   off += rank * vec;
    kdot = off; off += rpad * 4;
    qdot = off; off += rpad * 4;
    misc = off; off += 16;  // alpha, beta, k . q
    tv = align_up(off, 16);
  }
  __host__ __device__ int bytes(int depth, int ntv) const {
    return align_up(depth * slot + ntv * tv, 128);
  }
};

template <int BITS, int DK, bool DIAG, bool YOKED, int SLOT, int DEPTH>
__device__ __forceinline__ void lrb_issue_block(const BlockCursor<SLOT, DEPTH>& cur,
                                                const LrbParams& p, const LrbLayout& L,
                                                uint32_t ring16, uint32_t ring4, uint32_t code8,
                                                uint32_t shadow8, uint32_t uring, uint32_t tvs,
                                                int lane, int rr, int c, const uint8_t* codes_blk,
                                                const float* scales_l, unsigned sstride,
                                                const float* v_l, const float* shadow_blk,
                                                bool readout) {
  constexpr int LPR = DK / 32;
  constexpr int RW = 32 / LPR;
  constexpr int CB = 4 * BITS;
  constexpr unsigned CSTRIDE = RW * DK * BITS / 8;
  constexpr int O_SCALES = 32 * CB;
  constexpr int O_V = O_SCALES + 128;
  constexpr int VU = DK / 4;
  if (cur.tile_start) {
    __syncwarp();
    const uint32_t tv = tvs + cur.tv;
    const size_t t = cur.tile;
    if (lane < VU) {
      const uint32_t u = tv + static_cast<uint32_t>(vec_unit_offset(lane));
      cp16<0>(u + L.k, p.k + t * DK + 4 * lane);
      if (readout) cp16<0>(u + L.q, p.q + t * DK + 4 * lane);
      if constexpr (DIAG) cp16<0>(u + L.a, p.alpha + t * DK + 4 * lane);
    }
    if constexpr (!DIAG) {
      if (lane == 0) cp4<0>(tv + L.misc, p.alpha + t);
    }
    if (lane == 1) cp4<4>(tv + L.misc, p.beta + t);
    if (p.slot > 0) {
      // the accumulated decay and the buffered keys of this tile
      const int vec = (DK / 32) * kChunkStride * 4;
      if (lane < VU)
        cp16<0>(tv + L.A + static_cast<uint32_t>(vec_unit_offset(lane)), p.A_in + t * DK + 4 * lane);
      const float* kin = p.K_in + t * p.rank * DK;
      for (int i = lane; i < p.slot * VU; i += 32) {
        const int r = i / VU, u = i % VU;
        cp16<0>(tv + L.Kb + r * vec + static_cast<uint32_t>(vec_unit_offset(u)), kin + r * DK + 4 * u);
      }
    }
  }
  const uint32_t s4 = ring4 + cur.slot;
  const uint8_t* cs = codes_blk + static_cast<size_t>(cur.blk) * CSTRIDE;
  if constexpr (CB == 16) {
    cp16<0>(ring16 + cur.slot, cs);
  } else {
    cp16<0>(code8 + cur.slot, cs);
    cp16<256>(code8 + cur.slot, cs + 512);
  }
  cp4<O_SCALES>(s4, scales_l + static_cast<size_t>(cur.blk) * sstride);
  cp4<O_V>(s4, v_l + static_cast<size_t>(cur.blk) * RW);
  // this row's buffered coefficients U_r, r < slot: 16-byte units c, c+LPR, ...
  const int units = (p.slot + 3) >> 2;
  const float* urow = p.U + (static_cast<size_t>(cur.blk) * RW + rr) * p.rpad;
  for (int u = c; u < units; u += LPR) cp16<0>(uring + cur.slot + 16 * u, urow + 4 * u);
  if constexpr (YOKED) {
    constexpr int O_SHADOW = 0;  // offset added by the caller through shadow8
    const uint32_t d = shadow8 + cur.slot;
    const float* sh = shadow_blk + static_cast<size_t>(cur.blk) * (RW * DK);
    cp16<O_SHADOW + 0 * 4 * kShadowStride>(d, sh + 0 * 128);
    cp16<O_SHADOW + 1 * 4 * kShadowStride>(d, sh + 1 * 128);
    cp16<O_SHADOW + 2 * 4 * kShadowStride>(d, sh + 2 * 128);
    cp16<O_SHADOW + 3 * 4 * kShadowStride>(d, sh + 3 * 128);
    cp16<O_SHADOW + 4 * 4 * kShadowStride>(d, sh + 4 * 128);
    cp16<O_SHADOW + 5 * 4 * kShadowStride>(d, sh + 5 * 128);
    cp16<O_SHADOW + 6 * 4 * kShadowStride>(d, sh + 6 * 128);
    cp16<O_SHADOW + 7 * 4 * kShadowStride>(d, sh + 7 * 128);
  }
}

// The chunk's eight chains against another chunk, then the pairwise tree
// across the LPR lanes of the row: the fixed dot order.
template <int LPR>
__device__ __forceinline__ float chunk_dot(const float2 (&a)[16], const float2 (&b)[16]) {
  return row_tree<LPR>(chunk_sum(a, b));
}

// POLICY: 0 dynamic, 1 persistent, 2 yoked.  MERGE: last step of the period.
template <int BITS, int DK, int POLICY, bool BDR, bool DELTA, bool DIAG, bool MERGE, int DEPTH>
__global__ void __launch_bounds__(kStepThreads, ((POLICY == 2 || BDR || MERGE) ? QS_STEP_WARPS_PER_SM_LOW
                                                                              : QS_STEP_WARPS_PER_SM) /
                                                    kStepWarps)
    lrb_step_kernel(LrbParams p) {
  constexpr int LPR = DK / 32;
  constexpr int RW = 32 / LPR;
  constexpr int CW = BITS;
  constexpr int CB = 4 * BITS;
  constexpr bool YOKED = POLICY == 2;
  constexpr int QMAX = BITS == 4 ? 7 : 127;
  constexpr float kQf = static_cast<float>(QMAX);
  constexpr float kOff = kMagic + (BITS == 4 ? 8.0f : 128.0f);
  constexpr int WARPS = kStepWarps;
  constexpr unsigned CSTRIDE = RW * DK * BITS / 8;
  constexpr int O_SCALES = 32 * CB;
  constexpr int O_V = O_SCALES + 128;

  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31;
  const int warp = WARPS == 1 ? 0 : threadIdx.x >> 5;
  const int c = lane % LPR, rr = lane / LPR;
  const LrbLayout L(BITS, DK, DIAG, YOKED, MERGE, p.rank, p.rpad);
  // the ring slot size must be a compile-time multiple for the cursor: use
  // the runtime layout through a fixed upper bound of the slot size
  unsigned char* ring = smem + warp * p.warp_bytes;
  unsigned char* tvs = ring + DEPTH * L.slot;
  const uint32_t ring_s = smem_addr(ring);
  const uint32_t ring16 = ring_s + 16 * lane;
  const uint32_t ring4 = ring_s + 4 * lane;
  const uint32_t code8 = ring_s + 512 * (lane & 1) + 16 * (lane >> 1);
  const uint32_t shadow8 = ring_s + L.shadow + kShadowStride * (lane >> 3) + 16 * (lane & 7);
  const uint32_t uring = ring_s + L.u + rr * p.rpad * 4;
  const uint32_t tvs_s = smem_addr(tvs);
  const int tv_end = p.ntv * L.tv;
  const unsigned ng = DK / p.group;
  const unsigned g = (32 * c) / p.group;
  const bool readout = p.o != nullptr;
  const bool writes_scale = (32 * c) % p.group == 0;
  const int slot = p.slot;

  const long long gw = static_cast<long long>(blockIdx.x) * WARPS + warp;
  const long long nw = static_cast<long long>(gridDim.x) * WARPS;
  const unsigned b0 = static_cast<unsigned>(gw * p.nblocks / nw);
  const unsigned b1 = static_cast<unsigned>((gw + 1) * p.nblocks / nw);
  if (b0 >= b1) return;
  const unsigned bpt = static_cast<unsigned>(p.bpt);
  grid_dep_wait();
  grid_dep_launch();

  uint8_t* codes_l = p.codes + CB * lane;
  const uint8_t* codes_blk = p.codes + 16 * lane;
  const unsigned sstride = RW * ng;
  float* scales_l = p.scales + rr * ng + g;
  const float* v_l = p.v + rr;
  float* o_l = p.o + rr;
  float* shadow_l = p.shadow + rr * DK + 32 * c;
  const float* shadow_blk = p.shadow + 4 * lane;

  // The cursor advances ring slots by a runtime slot size: emulate with a
  // one-slot template size and scale the offset.
  BlockCursor<1, DEPTH> pre;
  pre.blk = b0;
  pre.tile = b0 / bpt;
  pre.next_tile = (pre.tile + 1) * bpt;
  pre.slot = 0;
  pre.tv = 0;
  pre.tile_start = true;
  BlockCursor<1, DEPTH> cur = pre;

  auto issue = [&](const BlockCursor<1, DEPTH>& x) {
    BlockCursor<1, DEPTH> y = x;
    y.slot = x.slot * L.slot;
    lrb_issue_block<BITS, DK, DIAG, YOKED, 1, DEPTH>(y, p, L, ring16, ring4, code8, shadow8, uring,
                                                   tvs_s, lane, rr, c, codes_blk, scales_l,
                                                   sstride, v_l, shadow_blk, readout);
  };

#pragma unroll
  for (int i = 0; i < DEPTH - 1; ++i) {
    if (pre.blk < b1) issue(pre);
    cp_async_commit();
    pre.advance(bpt, L.tv, tv_end);
  }

  float2 kk[16];
  float beta = 0.0f, a_scalar = 1.0f, kqn = 0.0f;

#pragma unroll 1
  for (; cur.blk < b1; cur.advance(bpt, L.tv, tv_end)) {
    __syncwarp();
    if (pre.blk < b1) issue(pre);
    cp_async_commit();
    pre.advance(bpt, L.tv, tv_end);
    cp_async_wait<DEPTH - 1>();
    __syncwarp();

    unsigned char* tv = tvs + cur.tv;
    if (cur.tile_start) {
      load_pairs(tv + L.k, c, kk);
      const float* misc = reinterpret_cast<const float*>(tv + L.misc);
      beta = misc[1];
      a_scalar = DIAG ? 1.0f : misc[0];
      const size_t t = cur.tile;
      const bool writer = !MERGE && cur.blk == cur.tile * bpt;
      // the decay of this step for this lane's chunk
      float2 aa[16];
      if constexpr (DIAG) {
        load_pairs(tv + L.a, c, aa);
      } else {
#pragma unroll
        for (int m = 0; m < 16; ++m) aa[m] = f2(a_scalar);
      }
      if (rr == 0) {
        // A = A_in * a for this chunk (A_in staged in the slot)
        float2 A[16];
        if (slot == 0) {
#pragma unroll
          for (int m = 0; m < 16; ++m) A[m] = aa[m];
        } else {
          load_pairs(tv + L.A, c, A);
#pragma unroll
          for (int m = 0; m < 16; ++m) A[m] = __fmul2_rn(A[m], aa[m]);
        }
        float* dA = reinterpret_cast<float*>(tv + L.A) + c * kChunkStride;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          dA[2 * m] = A[m].x;
          dA[2 * m + 1] = A[m].y;
        }
        if (writer) {
          float4* gA = reinterpret_cast<float4*>(p.A_out + t * DK + 32 * c);
          float4* gK = reinterpret_cast<float4*>(p.K_out + (t * p.rank + slot) * DK + 32 * c);
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            gA[m] = make_float4(A[2 * m].x, A[2 * m].y, A[2 * m + 1].x, A[2 * m + 1].y);
            gK[m] = make_float4(kk[2 * m].x, kk[2 * m].y, kk[2 * m + 1].x, kk[2 * m + 1].y);
          }
        }
      }
      if (readout) {
        float2 qq[16];
        load_pairs(tv + L.q, c, qq);
        kqn = chunk_dot<LPR>(kk, qq);
      }
      // decayed buffered keys and their products with k and q
      for (int r0 = 0; r0 < slot; r0 += RW) {
        const int r = r0 + rr;
        const bool live = r < slot;
        // K'_r = K_in_r * a (K_in_r staged in the slot; decayed in place below)
        float2 Kr[16];
        const int vec = LPR * kChunkStride * 4;
        load_pairs(tv + L.Kb + (live ? r : 0) * vec, c, Kr);
#pragma unroll
        for (int m = 0; m < 16; ++m) Kr[m] = live ? __fmul2_rn(Kr[m], aa[m]) : make_float2(0.0f, 0.0f);
        const float dk_ = chunk_dot<LPR>(Kr, kk);
        float dq_ = 0.0f;
        if (readout) {
          float2 qq[16];
          load_pairs(tv + L.q, c, qq);
          dq_ = chunk_dot<LPR>(Kr, qq);
        }
        if (live) {
          if (c == 0) {
            reinterpret_cast<float*>(tv + L.kdot)[r] = dk_;
            reinterpret_cast<float*>(tv + L.qdot)[r] = dq_;
          }
          {
            float* dK = reinterpret_cast<float*>(tv + L.Kb) + r * (LPR * kChunkStride) + c * kChunkStride;
#pragma unroll
            for (int m = 0; m < 16; ++m) {
              dK[2 * m] = Kr[m].x;
              dK[2 * m + 1] = Kr[m].y;
            }
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
    }
    const unsigned char* s = ring + cur.slot * L.slot;
    const size_t blk = cur.blk;
    const size_t row = blk * RW + rr;
    const float* ur = reinterpret_cast<const float*>(s + L.u) + rr * p.rpad;
    const float* kdot = reinterpret_cast<const float*>(tv + L.kdot);
    const float* qdot = reinterpret_cast<const float*>(tv + L.qdot);

    // ---- unpack and dequantize with the accumulated decay: S' = c * (s * A_j)
    uint32_t w[CW];
#pragma unroll
    for (int h = 0; h < CW / 4; ++h) {
      const uint4 u = reinterpret_cast<const uint4*>(s + h * 512)[lane];
      w[4 * h + 0] = u.x; w[4 * h + 1] = u.y; w[4 * h + 2] = u.z; w[4 * h + 3] = u.w;
    }
    const float s_old = reinterpret_cast<const float*>(s + O_SCALES)[lane];
    const float v_i = reinterpret_cast<const float*>(s + O_V)[lane];
    float2 Sp[16];
    decode_chunk<BITS>(w, Sp);
    float2 dref[(MERGE && BDR) ? 16 : 1];
    if constexpr (MERGE && BDR) {
#pragma unroll
      for (int m = 0; m < 16; ++m) dref[m] = __fmul2_rn(Sp[m], f2(s_old));
    }
    if constexpr (DIAG) {
      float2 A[16];
      load_pairs(tv + L.A, c, A);
#pragma unroll
      for (int m = 0; m < 16; ++m) Sp[m] = __fmul2_rn(Sp[m], __fmul2_rn(f2(s_old), A[m]));
    } else {
      // scalar decay: every A_j of the tile holds the same product of the
      // alphas, so s * A_j is one product per row (the same bits)
      const float sa = __fmul_rn(s_old, reinterpret_cast<const float*>(tv + L.A)[0]);
#pragma unroll
      for (int m = 0; m < 16; ++m) Sp[m] = __fmul2_rn(Sp[m], f2(sa));
    }

    // ---- the buffer's terms of u and o, U_ir kk_r and U_ir kq_r (r < slot),
    // continuing each chain from its dot product over S'
    float u_acc = 0.0f, o_acc = 0.0f;
    if (DELTA) u_acc = chunk_dot<LPR>(Sp, kk);
    float2 qq[16];
    if (readout && !MERGE) {
      load_pairs(tv + L.q, c, qq);
      o_acc = chunk_dot<LPR>(Sp, qq);
    }
    for (int r = 0; r < slot; ++r) {
      const float urr = ur[r];
      if (DELTA) u_acc = __fmaf_rn(urr, kdot[r], u_acc);
      if (readout && !MERGE) o_acc = __fmaf_rn(urr, qdot[r], o_acc);
    }

    // ---- write coefficient against S' + sum_r U_r K'_r^T
    float wcoef;
    if constexpr (DELTA) {
      wcoef = __fmul_rn(beta, __fsub_rn(v_i, u_acc));
    } else {
      wcoef = __fmul_rn(beta, v_i);
    }

    // ---- yoked shadow: the FP32 reference advances every step
    float m_shadow = 0.0f;
    if constexpr (YOKED) {
      float2 rs[16];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float4 t = reinterpret_cast<const float4*>(s + L.shadow + kShadowStride * lane)[u];
        rs[2 * u] = make_float2(t.x, t.y);
        rs[2 * u + 1] = make_float2(t.z, t.w);
      }
      if constexpr (DIAG) {
        float2 aa[16];
        load_pairs(tv + L.a, c, aa);
#pragma unroll
        for (int mm = 0; mm < 16; ++mm) rs[mm] = __fmul2_rn(rs[mm], aa[mm]);
      } else {
#pragma unroll
        for (int mm = 0; mm < 16; ++mm) rs[mm] = __fmul2_rn(rs[mm], f2(a_scalar));
      }
      float wr;
      if constexpr (DELTA) {
        wr = __fmul_rn(beta, __fsub_rn(v_i, chunk_dot<LPR>(rs, kk)));
      } else {
        wr = wcoef;
      }
#pragma unroll
      for (int mm = 0; mm < 16; ++mm) rs[mm] = __ffma2_rn(f2(wr), kk[mm], rs[mm]);
      float* rg = shadow_l + blk * (RW * DK);
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        uint32_t ww[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          ww[2 * e] = __float_as_uint(rs[4 * h + e].x);
          ww[2 * e + 1] = __float_as_uint(rs[4 * h + e].y);
        }
        st_global_v8(rg + 8 * h, ww);
      }
      m_shadow = row_max<LPR>(chunk_absmax(rs), p.group);
    }

    if constexpr (!MERGE) {
      // ---- bypass: the write joins the buffer, the stored state is kept
      if (readout) {
        const float o = __fmaf_rn(wcoef, kqn, o_acc);
        if (c == 0) o_l[blk * RW] = o;
      }
      if (c == 0) p.U[row * p.rpad + slot] = wcoef;
    } else {
      // ---- merge: x = S' + sum_r U_r K'_r^T + w k^T, requantized once
      float2 x[16], M[BDR ? 16 : 1];
#pragma unroll
      for (int m = 0; m < 16; ++m) x[m] = Sp[m];
      if constexpr (BDR) {
#pragma unroll
        for (int m = 0; m < 16; ++m) M[m] = make_float2(0.0f, 0.0f);
      }
      for (int r = 0; r < slot; ++r) {
        const float urr = ur[r];
        const float4* kr4 = reinterpret_cast<const float4*>(tv + L.Kb) + r * (LPR * kChunkStride / 4) +
                            c * (kChunkStride / 4);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const float4 t = kr4[m];
          x[2 * m] = __ffma2_rn(f2(urr), make_float2(t.x, t.y), x[2 * m]);
          x[2 * m + 1] = __ffma2_rn(f2(urr), make_float2(t.z, t.w), x[2 * m + 1]);
          if constexpr (BDR) {
            M[2 * m] = __ffma2_rn(f2(urr), make_float2(t.x, t.y), M[2 * m]);
            M[2 * m + 1] = __ffma2_rn(f2(urr), make_float2(t.z, t.w), M[2 * m + 1]);
          }
        }
      }
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        x[m] = __ffma2_rn(f2(wcoef), kk[m], x[m]);
        if constexpr (BDR) M[m] = __ffma2_rn(f2(wcoef), kk[m], M[m]);
      }
      if (readout) {
        float2 qq[16];
        load_pairs(tv + L.q, c, qq);
        const float o = chunk_dot<LPR>(x, qq);
        if (c == 0) o_l[blk * RW] = o;
      }
      float m = 0.0f;
      if constexpr (POLICY == 0) m = row_max<LPR>(chunk_absmax(x), p.group);
      if constexpr (POLICY == 2) m = m_shadow;
      float sp = POLICY == 1 ? s_old : div_qmax_fast<QMAX>(m);
      float inv = recip_fast(sp);
      bool normal = sp >= 0x1p-126f && sp < 0x1p126f;
      if constexpr (POLICY != 1) normal = normal && m <= 3.40282347e38f;
      bool zero = false;
      if (!normal) {
        if constexpr (POLICY != 1) sp = div_qmax_rn<QMAX>(m);
        zero = !(sp > 0.0f);
        inv = zero ? 0.0f : recip_rn(sp);
      }
      bool clamp;
      if constexpr (POLICY == 0) {
        clamp = !normal;
      } else {
        const float xm = chunk_absmax(x);
        clamp = !(__fmaf_rn(xm, inv, kOff) <= kOff + kQf);
      }
      float2 y[16];
      round_chunk<BITS>(x, inv, clamp, y);
      if (zero) {
#pragma unroll
        for (int mm = 0; mm < 16; ++mm) y[mm] = f2(kOff);
      }
      if constexpr (BDR) {
        if (!zero) {
          // sigma_j = sign of the accumulated update M_j
          float2 sg[16];
#pragma unroll
          for (int mm = 0; mm < 16; ++mm)
            sg[mm] = make_float2(M[mm].x > 0.0f ? 1.0f : (M[mm].x < 0.0f ? -1.0f : 0.0f),
                                 M[mm].y > 0.0f ? 1.0f : (M[mm].y < 0.0f ? -1.0f : 0.0f));
          bdr_chunk<BITS>(y, dref, sg, 1.0f, sp);
        }
      }
      uint32_t out[CW];
      pack_chunk<BITS>(y, out);
      uint8_t* cg = codes_l + blk * CSTRIDE;
      if constexpr (CW == 4) {
        *reinterpret_cast<uint4*>(cg) = make_uint4(out[0], out[1], out[2], out[3]);
      } else {
        st_global_v8(cg, out);
      }
      if constexpr (POLICY != 1) {
        if (writes_scale) scales_l[blk * sstride] = sp;
      }
    }
  }
  cp_async_wait<0>();
}

}  // namespace qs
