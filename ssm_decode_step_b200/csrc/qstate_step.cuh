// The fused decode step, organised per warp (sm_100a).
//
// The element-level definition (dequantize with the decayed scale, key
// projection, rank-1 write, readout, scale selection, rounding, packing) is
// the one of include/qstate.h and is shared with the rest of the library
// through the helpers of qstate_kernels.cuh; this file decides who computes
// which rows and how their bytes reach the registers.
//
// Work decomposition.  A row block is RW = 32 / (Dk/32) consecutive rows of
// one tile (8 rows for Dk = 128, 16 for Dk = 64); lane (rr, c) of a warp owns
// the 32-column chunk c of row rr of the block, so every reduction of the
// step is an in-lane chain plus log2(Dk/32) xor shuffles.  The row blocks of
// all tiles form one sequence, cut into one contiguous range per warp of the
// grid (sizes differ by at most one block), so the SMs get equal work
// whatever the tile count.  Warps never wait for each other: there is no
// block-level barrier in the kernel.
//
// Memory path.  A two-slot cp.async ring per warp holds the next row block
// while the current one is computed.  Every copy instruction reads 512
// consecutive bytes across the warp (lane l copies the l-th 16-byte unit
// of the block's codes or shadow, which may belong to another lane); the
// warp publishes a slot with __syncwarp after its cp.async.wait_group and
// again before the slot is refilled.  The per-tile vectors (k, q, diagonal
// alpha, alpha, beta, sign(k) for BDR) go once per tile into one of `ntv`
// per-warp slots; ntv covers every tile that the prefetch window can span.
// New codes, scales, shadow and o leave straight from registers with
// 16/32-byte stores.  One warp per CTA by default, so the row-block cursor
// is uniform across the CTA.
#pragma once

#include "qstate_kernels.cuh"

namespace qs {

// Ring depth (row blocks per lane in the ring) of the non-yoked and the
// yoked kernels.
#ifndef QS_DEPTH
#define QS_DEPTH 2
#endif
#ifndef QS_DEPTH_YOKED
#define QS_DEPTH_YOKED 2
#endif
// Warps per CTA of the step kernel.  With one, everything derived from the
// row-block cursor is uniform across the CTA, which the compiler keeps in
// uniform registers and branches on without divergence bookkeeping.
#ifndef QS_STEP_WARPS
#define QS_STEP_WARPS 1
#endif
constexpr int kStepWarps = QS_STEP_WARPS;
constexpr int kStepThreads = 32 * kStepWarps;
// Resident warps per SM the register allocation targets.
#ifndef QS_STEP_WARPS_PER_SM
#define QS_STEP_WARPS_PER_SM 16
#endif
#ifndef QS_STEP_WARPS_PER_SM_LOW
#define QS_STEP_WARPS_PER_SM_LOW 12
#endif

struct WarpStepParams {
  uint8_t* codes;
  float* scales;
  float* shadow;
  const float* q;
  const float* k;
  const float* v;
  const float* alpha;
  const float* beta;
  float* o;
  int nblocks;     // row blocks in all tiles: tiles * dv / RW
  int bpt;         // row blocks per tile: dv / RW
  int group;
  int ntv;         // tile-vector slots per warp
  int warp_bytes;  // shared memory per warp
};

// Bytes per lane of a ring slot's shadow array: the lane's 128 bytes plus
// 16 of padding, so that the lanes of a quarter-warp read 8 different
// 16-byte bank groups.
constexpr int kShadowStride = 144;

// One warp's shared memory: DEPTH ring slots, then ntv tile-vector slots.
// Within a ring slot the codes are [16-byte unit][lane] and the scales and
// v are [lane], so that 32 lanes reading their own element of one array
// touch consecutive words (no bank conflicts); the shadow is [lane][144 B].
struct WarpLayout {
  int slot, codes, scales, v, shadow;  // ring slot size and offsets
  int tv, k, q, a, sk, misc;           // tile-vector slot size and offsets

  __host__ __device__ WarpLayout(int bits, int dk, bool diag, bool bdr, bool yoked) {
    int off = 0;
    codes = off;  off += 32 * 4 * bits;
    scales = off; off += 32 * 4;
    v = off;      off += 32 * 4;
    shadow = off; off += yoked ? 32 * kShadowStride : 0;
    slot = off;
    const int vec = (dk / 32) * kChunkStride * 4;
    off = 0;
    k = off;    off += vec;
    q = off;    off += vec;
    a = off;    off += diag ? vec : 0;
    sk = off;   off += bdr ? vec : 0;
    misc = off; off += 16;
    tv = off;
  }
  __host__ __device__ int bytes(int depth, int ntv) const {
    return align_up(depth * slot + ntv * tv, 128);
  }
};

// 32-bit shared-memory addresses and cp.async with an immediate offset.
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
template <int OFF>
__device__ __forceinline__ void cp16(uint32_t s, const void* g) {
  asm volatile("cp.async.cg.shared.global [%0+%2], [%1], 16;\n" ::"r"(s), "l"(g), "n"(OFF) : "memory");
}
template <int OFF>
__device__ __forceinline__ void cp4(uint32_t s, const void* g) {
  asm volatile("cp.async.ca.shared.global [%0+%2], [%1], 4;\n" ::"r"(s), "l"(g), "n"(OFF) : "memory");
}

// The fast forms of the scale arithmetic, exact on their ranges: m / qmax
// for finite m >= 0, and 1 / s for s in [2^-126, 2^126) (the branch-free
// parts of div_qmax_rn and recip_rn; the step checks the ranges once per
// chunk and otherwise takes the general path).
template <int Q>
__device__ __forceinline__ float div_qmax_fast(float m) {
  constexpr float r = 1.0f / static_cast<float>(Q);
  const float q0 = __fmul_rn(m, r);
  const float rem = __fmaf_rn(-q0, static_cast<float>(Q), m);
  return __fmaf_rn(rem, r, q0);
}
__device__ __forceinline__ float recip_fast(float s) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(s));
  const float e = __fmaf_rn(-s, y, 1.0f);
  return __fmaf_rn(y, e, y);
}

// Cursor over one warp's row blocks: block index, tile, ring-slot byte
// offset and tile-vector-slot byte offset, advanced without divisions.
template <int SLOT, int DEPTH>
struct BlockCursor {
  unsigned blk, tile, next_tile;
  int slot, tv;
  bool tile_start;
  __device__ __forceinline__ void advance(unsigned bpt, int tv_bytes, int tv_end) {
    ++blk;
    slot += SLOT;
    if (slot == SLOT * DEPTH) slot = 0;
    tile_start = blk == next_tile;
    if (tile_start) {
      ++tile;
      next_tile += bpt;
      tv += tv_bytes;
      if (tv == tv_end) tv = 0;
    }
  }
};

// Issue the copies of row block cur.blk into ring slot cur.slot (ring16,
// ring4, code8, shadow8: this lane's destinations in slot 0) and, at a tile
// start, the tile's vectors into the warp's slot cur.tv.
template <int BITS, int DK, bool DIAG, bool YOKED, int SLOT, int DEPTH, bool UPDATE = true>
__device__ __forceinline__ void issue_block(const BlockCursor<SLOT, DEPTH>& cur, const WarpStepParams& p,
                                            const WarpLayout& L, uint32_t ring16, uint32_t ring4,
                                            uint32_t code8, uint32_t shadow8, uint32_t tvs, int lane,
                                            const uint8_t* codes_blk, const float* scales_l,
                                            unsigned sstride, const float* v_l,
                                            const float* shadow_blk, bool readout) {
  constexpr int LPR = DK / 32;
  constexpr int RW = 32 / LPR;
  constexpr int CB = 4 * BITS;
  constexpr unsigned CSTRIDE = RW * DK * BITS / 8;
  constexpr int O_SCALES = 32 * CB;
  constexpr int O_V = O_SCALES + 128;
  constexpr int O_SHADOW = O_V + 128;
  constexpr int VU = DK / 4;  // 16-byte units per Dk vector
  static_assert(RW * DK * 4 == 8 * 512, "a row block's shadow is eight 512-byte copies");
  if (cur.tile_start) {
    // other lanes may still read the tile vectors that this slot held
    __syncwarp();
    const uint32_t tv = tvs + cur.tv;
    const size_t t = cur.tile;
    if (lane < VU) {
      const uint32_t u = tv + static_cast<uint32_t>(vec_unit_offset(lane));
      if constexpr (UPDATE) cp16<0>(u + L.k, p.k + t * DK + 4 * lane);
      if (readout) cp16<0>(u + L.q, p.q + t * DK + 4 * lane);
      if constexpr (UPDATE && DIAG) cp16<0>(u + L.a, p.alpha + t * DK + 4 * lane);
    }
    if constexpr (UPDATE && !DIAG) {
      if (lane == 0) cp4<0>(tv + L.misc, p.alpha + t);
    }
    if constexpr (UPDATE) {
      if (lane == 1) cp4<4>(tv + L.misc, p.beta + t);
    }
  }
  // Every copy instruction below reads 512 consecutive bytes across the
  // warp: lane l copies the l-th 16-byte unit, which may belong to another
  // lane (the compute loop publishes the slot with __syncwarp).
  const uint32_t s4 = ring4 + cur.slot;
  const uint8_t* cs = codes_blk + static_cast<size_t>(cur.blk) * CSTRIDE;
  if constexpr (CB == 16) {
    cp16<0>(ring16 + cur.slot, cs);
  } else {
    // unit G = 32 h + lane is half G & 1 of lane G >> 1's 32 bytes
    cp16<0>(code8 + cur.slot, cs);
    cp16<256>(code8 + cur.slot, cs + 512);
  }
  cp4<O_SCALES>(s4, scales_l + static_cast<size_t>(cur.blk) * sstride);
  if constexpr (UPDATE) cp4<O_V>(s4, v_l + static_cast<size_t>(cur.blk) * RW);
  if constexpr (YOKED) {
    // unit G = 32 i + lane is unit G & 7 of lane G >> 3's 128 bytes
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

// POLICY: 0 dynamic, 1 persistent, 2 yoked.
template <int BITS, int DK, int POLICY, bool BDR, bool DELTA, bool DIAG, int DEPTH>
__global__ void __launch_bounds__(kStepThreads, ((POLICY == 2 || BDR) ? QS_STEP_WARPS_PER_SM_LOW
                                                                    : QS_STEP_WARPS_PER_SM) / kStepWarps)
    step_kernel(WarpStepParams p) {
  constexpr int LPR = DK / 32;
  constexpr int RW = 32 / LPR;
  constexpr int CW = BITS;      // 32-bit code words per lane
  constexpr int CB = 4 * BITS;  // code bytes per lane
  constexpr bool YOKED = POLICY == 2;
  constexpr int QMAX = BITS == 4 ? 7 : 127;
  constexpr float kQf = static_cast<float>(QMAX);
  constexpr float kOff = kMagic + (BITS == 4 ? 8.0f : 128.0f);
  constexpr int WARPS = kStepWarps;
  constexpr unsigned CSTRIDE = RW * DK * BITS / 8;  // code bytes per row block
  // ring-slot layout in bytes (the same as WarpLayout's)
  constexpr int O_SCALES = 32 * CB;
  constexpr int O_V = O_SCALES + 128;
  constexpr int O_SHADOW = O_V + 128;
  constexpr int SLOT = O_SHADOW + (YOKED ? 32 * kShadowStride : 0);

  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31;
  const int warp = WARPS == 1 ? 0 : threadIdx.x >> 5;
  const int c = lane % LPR, rr = lane / LPR;
  const WarpLayout L(BITS, DK, DIAG, BDR, YOKED);
  unsigned char* ring = smem + warp * p.warp_bytes;
  unsigned char* tvs = ring + DEPTH * SLOT;
  const uint32_t ring16 = smem_addr(ring) + 16 * lane;
  const uint32_t ring4 = smem_addr(ring) + 4 * lane;
  const uint32_t code8 = smem_addr(ring) + 512 * (lane & 1) + 16 * (lane >> 1);
  const uint32_t shadow8 = smem_addr(ring) + kShadowStride * (lane >> 3) + 16 * (lane & 7);
  const uint32_t tvs_s = smem_addr(tvs);
  const int tv_end = p.ntv * L.tv;
  const unsigned ng = DK / p.group;
  const unsigned g = (32 * c) / p.group;
  const bool readout = p.o != nullptr;
  const bool writes_scale = (32 * c) % p.group == 0;

  // this warp's contiguous range of row blocks
  const long long gw = static_cast<long long>(blockIdx.x) * WARPS + warp;
  const long long nw = static_cast<long long>(gridDim.x) * WARPS;
  const unsigned b0 = static_cast<unsigned>(gw * p.nblocks / nw);
  const unsigned b1 = static_cast<unsigned>((gw + 1) * p.nblocks / nw);
  if (b0 >= b1) return;  // warp-uniform; nothing in this kernel waits for other warps
  const unsigned bpt = static_cast<unsigned>(p.bpt);
  grid_dep_wait();
  grid_dep_launch();

  // per-lane bases; row block blk adds blk times a per-block stride
  uint8_t* codes_l = p.codes + CB * lane;
  const uint8_t* codes_blk = p.codes + 16 * lane;
  const float* shadow_blk = p.shadow + 4 * lane;
  const unsigned sstride = RW * ng;
  float* scales_l = p.scales + rr * ng + g;
  const float* v_l = p.v + rr;
  float* o_l = p.o + rr;
  float* shadow_l = p.shadow + rr * DK + 32 * c;

  BlockCursor<SLOT, DEPTH> pre;
  pre.blk = b0;
  pre.tile = b0 / bpt;
  pre.next_tile = (pre.tile + 1) * bpt;
  pre.slot = 0;
  pre.tv = 0;
  pre.tile_start = true;
  BlockCursor<SLOT, DEPTH> cur = pre;

#pragma unroll
  for (int i = 0; i < DEPTH - 1; ++i) {
    if (pre.blk < b1)
      issue_block<BITS, DK, DIAG, YOKED>(pre, p, L, ring16, ring4, code8, shadow8, tvs_s, lane,
                                         codes_blk, scales_l, sstride, v_l, shadow_blk, readout);
    cp_async_commit();
    pre.advance(bpt, L.tv, tv_end);
  }

  float2 kk[16];
  float beta = 0.0f, a_scalar = 1.0f;

#pragma unroll 1
  for (; cur.blk < b1; cur.advance(bpt, L.tv, tv_end)) {
    // all lanes are done with the slot that the next copies overwrite
    if constexpr (CB == 32 || YOKED) __syncwarp();
    if (pre.blk < b1)
      issue_block<BITS, DK, DIAG, YOKED>(pre, p, L, ring16, ring4, code8, shadow8, tvs_s, lane,
                                         codes_blk, scales_l, sstride, v_l, shadow_blk, readout);
    cp_async_commit();
    pre.advance(bpt, L.tv, tv_end);
    cp_async_wait<DEPTH - 1>();
    // every lane's copies for this block have landed: publish them
    if constexpr (CB == 32 || YOKED) __syncwarp();

    unsigned char* tv = tvs + cur.tv;
    if (cur.tile_start) {
      // every lane's copies of the tile vectors have landed: publish them
      __syncwarp();
      load_pairs(tv + L.k, c, kk);
      const float* misc = reinterpret_cast<const float*>(tv + L.misc);
      beta = misc[1];
      a_scalar = DIAG ? 1.0f : misc[0];
      if constexpr (BDR) {
        // sign(k_j) per column, in the layout of k
        if (rr == 0) {
          float* ss = reinterpret_cast<float*>(tv + L.sk) + c * kChunkStride;
          float2 kt[16];
          load_pairs(tv + L.k, c, kt);
#pragma unroll
          for (int m = 0; m < 16; ++m) {
            const float2 kv = kt[m];
            ss[2 * m] = kv.x > 0.0f ? 1.0f : (kv.x < 0.0f ? -1.0f : 0.0f);
            ss[2 * m + 1] = kv.y > 0.0f ? 1.0f : (kv.y < 0.0f ? -1.0f : 0.0f);
          }
        }
        __syncwarp();
      }
    }
    const unsigned char* s = ring + cur.slot;
    const size_t blk = cur.blk;

    // ---- a1: unpack this lane's 32 codes
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
    // BDR's reference: the element as stored before the step, d = c * s
    float2 dref[BDR ? 16 : 1];
    if constexpr (BDR) {
#pragma unroll
      for (int m = 0; m < 16; ++m) dref[m] = __fmul2_rn(Sp[m], f2(s_old));
    }

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
      wcoef = __fmul_rn(beta, __fsub_rn(v_i, row_tree<LPR>(chunk_sum(Sp, kk))));
    } else {
      wcoef = __fmul_rn(beta, v_i);
    }
    float2 x[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) x[m] = __ffma2_rn(f2(wcoef), kk[m], Sp[m]);

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
      if (c == 0) o_l[blk * RW] = o;
    }

    // ---- a6/a7: scale selection (yoked: shadow update first)
    float m = 0.0f;  // group max of |x| (dynamic) or |R| (yoked)
    if constexpr (POLICY == 0) {
      m = row_max<LPR>(chunk_absmax(x), p.group);
    } else if constexpr (POLICY == 2) {
      float2 rs[16];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float4 t = reinterpret_cast<const float4*>(s + O_SHADOW + kShadowStride * lane)[u];
        rs[2 * u] = make_float2(t.x, t.y);
        rs[2 * u + 1] = make_float2(t.z, t.w);
      }
      // R' = R * a
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
        wr = __fmul_rn(beta, __fsub_rn(v_i, row_tree<LPR>(chunk_sum(rs, kk))));
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
      m = row_max<LPR>(chunk_absmax(rs), p.group);
    }

    // ---- a8/a9: round (and BDR), pack, store codes (and scales)
    // The scale and its reciprocal come from the fast forms when the group
    // max is finite and the scale lies in [2^-126, 2^126) (both are then
    // exact); any other chunk takes the general routines and the zero-scale
    // rule.  Rounding then runs once, followed by clamping only where some
    // element can leave [-qmax, qmax].
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
      // |x| <= group max, so |x * inv| <= qmax (1 + 2^-23) rounds inside
      // the range whenever the scale is a normal float below 2^126
      clamp = !normal;
    } else {
      const float xm = chunk_absmax(x);
      clamp = !(__fmaf_rn(xm, inv, kOff) <= kOff + kQf);
    }
    float2 y[16];
    round_chunk<BITS>(x, inv, clamp, y);
    if (zero) {
      // zero-scale rule: every code of the group is 0
#pragma unroll
      for (int mm = 0; mm < 16; ++mm) y[mm] = f2(kOff);
    }
    if constexpr (BDR) {
      float2 sk[16];
      load_pairs(tv + L.sk, c, sk);
      const float sw = zero ? 0.0f : (wcoef > 0.0f ? 1.0f : (wcoef < 0.0f ? -1.0f : 0.0f));
      bdr_chunk<BITS>(y, dref, sk, sw, sp);
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
  cp_async_wait<0>();
}

// Readout of the stored state without changing it (qstate_readout):
// o_i = d_i . q with d = c * s, on the step kernel's layout (row-block
// ranges per warp, the ring carrying codes and scales, q once per tile).
template <int BITS, int DK, int DEPTH>
__global__ void __launch_bounds__(kStepThreads, QS_STEP_WARPS_PER_SM / kStepWarps)
    readout_kernel(WarpStepParams p) {
  constexpr int LPR = DK / 32;
  constexpr int RW = 32 / LPR;
  constexpr int CW = BITS;
  constexpr int CB = 4 * BITS;
  constexpr int WARPS = kStepWarps;
  constexpr int O_SCALES = 32 * CB;
  constexpr int O_V = O_SCALES + 128;
  constexpr int SLOT = O_V + 128;

  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31;
  const int warp = WARPS == 1 ? 0 : threadIdx.x >> 5;
  const int c = lane % LPR, rr = lane / LPR;
  const WarpLayout L(BITS, DK, false, false, false);
  unsigned char* ring = smem + warp * p.warp_bytes;
  unsigned char* tvs = ring + DEPTH * SLOT;
  const uint32_t ring16 = smem_addr(ring) + 16 * lane;
  const uint32_t ring4 = smem_addr(ring) + 4 * lane;
  const uint32_t code8 = smem_addr(ring) + 512 * (lane & 1) + 16 * (lane >> 1);
  const uint32_t tvs_s = smem_addr(tvs);
  const int tv_end = p.ntv * L.tv;
  const unsigned ng = DK / p.group;
  const unsigned g = (32 * c) / p.group;

  const long long gw = static_cast<long long>(blockIdx.x) * WARPS + warp;
  const long long nw = static_cast<long long>(gridDim.x) * WARPS;
  const unsigned b0 = static_cast<unsigned>(gw * p.nblocks / nw);
  const unsigned b1 = static_cast<unsigned>((gw + 1) * p.nblocks / nw);
  if (b0 >= b1) return;
  const unsigned bpt = static_cast<unsigned>(p.bpt);
  grid_dep_wait();
  grid_dep_launch();
  const uint8_t* codes_blk = p.codes + 16 * lane;
  const unsigned sstride = RW * ng;
  const float* scales_l = p.scales + rr * ng + g;
  float* o_l = p.o + rr;

  BlockCursor<SLOT, DEPTH> pre;
  pre.blk = b0;
  pre.tile = b0 / bpt;
  pre.next_tile = (pre.tile + 1) * bpt;
  pre.slot = 0;
  pre.tv = 0;
  pre.tile_start = true;
  BlockCursor<SLOT, DEPTH> cur = pre;
#pragma unroll
  for (int i = 0; i < DEPTH - 1; ++i) {
    if (pre.blk < b1)
      issue_block<BITS, DK, false, false, SLOT, DEPTH, false>(pre, p, L, ring16, ring4, code8, 0u, tvs_s,
                                                              lane, codes_blk, scales_l, sstride,
                                                              nullptr, nullptr, true);
    cp_async_commit();
    pre.advance(bpt, L.tv, tv_end);
  }
  float2 qq[16];
#pragma unroll 1
  for (; cur.blk < b1; cur.advance(bpt, L.tv, tv_end)) {
    if constexpr (CB == 32) __syncwarp();
    if (pre.blk < b1)
      issue_block<BITS, DK, false, false, SLOT, DEPTH, false>(pre, p, L, ring16, ring4, code8, 0u, tvs_s,
                                                              lane, codes_blk, scales_l, sstride,
                                                              nullptr, nullptr, true);
    cp_async_commit();
    pre.advance(bpt, L.tv, tv_end);
    cp_async_wait<DEPTH - 1>();
    if constexpr (CB == 32) __syncwarp();
    const unsigned char* tv = tvs + cur.tv;
    if (cur.tile_start) {
      __syncwarp();
      load_pairs(tv + L.q, c, qq);
    }
    const unsigned char* s = ring + cur.slot;
    uint32_t w[CW];
#pragma unroll
    for (int h = 0; h < CW / 4; ++h) {
      const uint4 u = reinterpret_cast<const uint4*>(s + h * 512)[lane];
      w[4 * h + 0] = u.x; w[4 * h + 1] = u.y; w[4 * h + 2] = u.z; w[4 * h + 3] = u.w;
    }
    const float sc = reinterpret_cast<const float*>(s + O_SCALES)[lane];
    float2 d[16];
    decode_chunk<BITS>(w, d);
    ChunkDot acc;
#pragma unroll
    for (int m = 0; m < 16; ++m) acc.add(m, __fmul2_rn(d[m], f2(sc)), qq[m]);
    const float o = row_tree<LPR>(acc.sum());
    if (c == 0) o_l[static_cast<size_t>(cur.blk) * RW] = o;
  }
  cp_async_wait<0>();
}

}  // namespace qs
