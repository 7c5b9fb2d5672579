// The C ABI of include/qstate.h: argument validation and dispatch to the
// compile-time kernel instances.  No memory is allocated here; the only
// process-wide state is the per-device SM count and the once-per-kernel
// shared-memory attribute.
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/qstate.h"
#include "qstate_fp32.cuh"
#include "qstate_launch.h"
#include "qstate_launch_prefill.h"
#include "qstate_norms.cuh"

namespace qs {

int device_sm_count() {
  static std::mutex mu;
  static int counts[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
  std::lock_guard<std::mutex> lock(mu);
  if (counts[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 1;
    counts[dev] = n;
  }
  return counts[dev];
}

// ---------------------------------------------------------------------------
// self-check of the fast arithmetic against the IEEE routines
// ---------------------------------------------------------------------------
// Every float bit pattern in [lo, hi): recip_rn against __frcp_rn on its
// fast range, and div_qmax_rn<7>, <127> against __fdiv_rn on all finite
// non-negative values.  Mismatch counts are added to bad[0..2].
__global__ void selfcheck_kernel(unsigned long long* bad, uint32_t lo, uint32_t hi) {
  unsigned long long b0 = 0, b1 = 0, b2 = 0;
  for (uint64_t i = lo + static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < hi;
       i += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
    const float x = __uint_as_float(static_cast<uint32_t>(i));
    if (!(x >= 0.0f) || x > 3.40282347e38f) continue;
    if (x >= 0x1p-126f && x < 0x1p126f) b0 += __float_as_uint(recip_rn(x)) != __float_as_uint(__frcp_rn(x));
    b1 += __float_as_uint(div_qmax_rn<7>(x)) != __float_as_uint(__fdiv_rn(x, 7.0f));
    b2 += __float_as_uint(div_qmax_rn<127>(x)) != __float_as_uint(__fdiv_rn(x, 127.0f));
  }
  if (b0) atomicAdd(&bad[0], b0);
  if (b1) atomicAdd(&bad[1], b1);
  if (b2) atomicAdd(&bad[2], b2);
}

}  // namespace qs

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Range {
  uintptr_t lo, hi;  // [lo, hi)
};

Range range_of(const void* p, size_t bytes) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
  return {lo, lo + bytes};
}

bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi && a.hi > a.lo && b.hi > b.lo; }

// Field ranges of the configuration; 0 = fine, else the status to return.
qs_status check_config(const qs_config* c) {
  if (c == nullptr) return QS_ERR_INVALID_ARG;
  if (c->num_tiles < 0) return QS_ERR_INVALID_ARG;
  if (c->dk < 1 || c->dv < 1) return QS_ERR_INVALID_ARG;
  if (c->bits != 4 && c->bits != 8) return QS_ERR_INVALID_ARG;
  if (c->group < 1 || c->dk % c->group != 0) return QS_ERR_INVALID_ARG;
  if (c->delta != 0 && c->delta != 1) return QS_ERR_INVALID_ARG;
  if (c->decay != QS_DECAY_SCALAR && c->decay != QS_DECAY_DIAGONAL) return QS_ERR_INVALID_ARG;
  if (c->policy != QS_SCALE_DYNAMIC && c->policy != QS_SCALE_PERSISTENT && c->policy != QS_SCALE_YOKED)
    return QS_ERR_INVALID_ARG;
  if (c->rounding != QS_ROUND_NEAREST && c->rounding != QS_ROUND_BDR) return QS_ERR_INVALID_ARG;
  // what this build has kernels for
  if (c->dk != 64 && c->dk != 128) return QS_ERR_UNSUPPORTED;
  if (c->dv % 16 != 0 || c->dv > 4096) return QS_ERR_UNSUPPORTED;
  if (static_cast<long long>(c->num_tiles) * (c->dv / 8) > 0x7fffffffLL) return QS_ERR_UNSUPPORTED;
  if (c->group != 32 && c->group != 64 && c->group != 128) return QS_ERR_UNSUPPORTED;
  return QS_OK;
}

struct Sizes {
  size_t codes, scales, shadow, vec_k, vec_v, alpha, tile_scalars;
};

Sizes sizes_of(const qs_config* c) {
  const size_t T = static_cast<size_t>(c->num_tiles);
  Sizes s;
  s.codes = T * c->dv * c->dk * c->bits / 8;
  s.scales = T * c->dv * (c->dk / c->group) * sizeof(float);
  s.shadow = c->policy == QS_SCALE_YOKED ? T * c->dv * c->dk * sizeof(float) : 0;
  s.vec_k = T * c->dk * sizeof(float);
  s.vec_v = T * c->dv * sizeof(float);
  s.alpha = c->decay == QS_DECAY_DIAGONAL ? s.vec_k : T * sizeof(float);
  s.tile_scalars = T * sizeof(float);
  return s;
}

qs_status from_cuda(cudaError_t e) { return e == cudaSuccess ? QS_OK : QS_ERR_CUDA; }

// Written buffers must not overlap each other or any input.
bool any_overlap(const Range* written, int nw, const Range* read, int nr) {
  for (int i = 0; i < nw; ++i) {
    for (int j = i + 1; j < nw; ++j)
      if (overlap(written[i], written[j])) return true;
    for (int j = 0; j < nr; ++j)
      if (overlap(written[i], read[j])) return true;
  }
  return false;
}

template <int BITS, int DK>
cudaError_t dispatch_step(const qs_config* c, const qs::StepParams& p, cudaStream_t s) {
  const bool bdr = c->rounding == QS_ROUND_BDR, delta = c->delta == 1, diag = c->decay == QS_DECAY_DIAGONAL;
  const int sel = (c->policy * 8) + (bdr ? 4 : 0) + (delta ? 2 : 0) + (diag ? 1 : 0);
  using namespace qs;
  switch (sel) {
#define QS_CASE(P, R, DE, DI) \
  case (P * 8 + R * 4 + DE * 2 + DI): return launch_step<BITS, DK, P, R, DE, DI>(p, s);
    QS_CASE(0, 0, 0, 0) QS_CASE(0, 0, 0, 1) QS_CASE(0, 0, 1, 0) QS_CASE(0, 0, 1, 1)
    QS_CASE(0, 1, 0, 0) QS_CASE(0, 1, 0, 1) QS_CASE(0, 1, 1, 0) QS_CASE(0, 1, 1, 1)
    QS_CASE(1, 0, 0, 0) QS_CASE(1, 0, 0, 1) QS_CASE(1, 0, 1, 0) QS_CASE(1, 0, 1, 1)
    QS_CASE(1, 1, 0, 0) QS_CASE(1, 1, 0, 1) QS_CASE(1, 1, 1, 0) QS_CASE(1, 1, 1, 1)
    QS_CASE(2, 0, 0, 0) QS_CASE(2, 0, 0, 1) QS_CASE(2, 0, 1, 0) QS_CASE(2, 0, 1, 1)
    QS_CASE(2, 1, 0, 0) QS_CASE(2, 1, 0, 1) QS_CASE(2, 1, 1, 0) QS_CASE(2, 1, 1, 1)
#undef QS_CASE
    default: return cudaErrorInvalidValue;
  }
}

template <int BITS, int DK>
cudaError_t dispatch_lrb(const qs_config* c, const qs::LrbParams& p, bool merge, cudaStream_t s) {
  using namespace qs;
  const bool bdr = c->rounding == QS_ROUND_BDR, delta = c->delta == 1, diag = c->decay == QS_DECAY_DIAGONAL;
  const int T = c->num_tiles, dv = c->dv;
  if (!merge) {
    const int sel = (c->policy == QS_SCALE_YOKED ? 4 : 0) + (delta ? 2 : 0) + (diag ? 1 : 0);
    switch (sel) {
      case 0: return launch_lrb<BITS, DK, 0, false, false, false, false>(p, T, dv, s);
      case 1: return launch_lrb<BITS, DK, 0, false, false, true, false>(p, T, dv, s);
      case 2: return launch_lrb<BITS, DK, 0, false, true, false, false>(p, T, dv, s);
      case 3: return launch_lrb<BITS, DK, 0, false, true, true, false>(p, T, dv, s);
      case 4: return launch_lrb<BITS, DK, 2, false, false, false, false>(p, T, dv, s);
      case 5: return launch_lrb<BITS, DK, 2, false, false, true, false>(p, T, dv, s);
      case 6: return launch_lrb<BITS, DK, 2, false, true, false, false>(p, T, dv, s);
      default: return launch_lrb<BITS, DK, 2, false, true, true, false>(p, T, dv, s);
    }
  }
  const int sel = (c->policy * 8) + (bdr ? 4 : 0) + (delta ? 2 : 0) + (diag ? 1 : 0);
  switch (sel) {
#define QS_CASE(P, R, DE, DI) \
  case (P * 8 + R * 4 + DE * 2 + DI): return launch_lrb<BITS, DK, P, R, DE, DI, true>(p, T, dv, s);
    QS_CASE(0, 0, 0, 0) QS_CASE(0, 0, 0, 1) QS_CASE(0, 0, 1, 0) QS_CASE(0, 0, 1, 1)
    QS_CASE(0, 1, 0, 0) QS_CASE(0, 1, 0, 1) QS_CASE(0, 1, 1, 0) QS_CASE(0, 1, 1, 1)
    QS_CASE(1, 0, 0, 0) QS_CASE(1, 0, 0, 1) QS_CASE(1, 0, 1, 0) QS_CASE(1, 0, 1, 1)
    QS_CASE(1, 1, 0, 0) QS_CASE(1, 1, 0, 1) QS_CASE(1, 1, 1, 0) QS_CASE(1, 1, 1, 1)
    QS_CASE(2, 0, 0, 0) QS_CASE(2, 0, 0, 1) QS_CASE(2, 0, 1, 0) QS_CASE(2, 0, 1, 1)
    QS_CASE(2, 1, 0, 0) QS_CASE(2, 1, 0, 1) QS_CASE(2, 1, 1, 0) QS_CASE(2, 1, 1, 1)
#undef QS_CASE
    default: return cudaErrorInvalidValue;
  }
}

int lrb_rpad(int rank) { return (rank + 3) / 4 * 4; }

}  // namespace

extern "C" {

int qstate_version(void) { return 100; }

qs_status qstate_selfcheck(unsigned long long* mismatches, cudaStream_t stream) {
  if (mismatches == nullptr || !aligned(mismatches, 8)) return QS_ERR_INVALID_ARG;
  cudaError_t e = cudaMemsetAsync(mismatches, 0, 3 * sizeof(unsigned long long), stream);
  if (e != cudaSuccess) return QS_ERR_CUDA;
  // all non-negative finite float bit patterns
  qs::selfcheck_kernel<<<qs::device_sm_count() * 16, 256, 0, stream>>>(mismatches, 0u, 0x7F800000u);
  return from_cuda(cudaGetLastError());
}

const char* qstate_status_string(qs_status s) {
  switch (s) {
    case QS_OK: return "ok";
    case QS_ERR_INVALID_ARG: return "invalid argument";
    case QS_ERR_UNSUPPORTED: return "configuration not supported by this build";
    case QS_ERR_CUDA: return "CUDA launch error";
  }
  return "unknown status";
}

qs_status qstate_query_sizes(const qs_config* cfg, size_t* codes_bytes, size_t* scales_bytes,
                             size_t* shadow_bytes) {
  const qs_status st = check_config(cfg);
  if (st != QS_OK) return st;
  const Sizes s = sizes_of(cfg);
  if (codes_bytes) *codes_bytes = s.codes;
  if (scales_bytes) *scales_bytes = s.scales;
  if (shadow_bytes) *shadow_bytes = s.shadow;
  return QS_OK;
}

qs_status qstate_init(const qs_config* cfg, const float* S0, void* codes, float* scales,
                      float* shadow, cudaStream_t stream) {
  qs_status st = check_config(cfg);
  if (st != QS_OK) return st;
  const bool yoked = cfg->policy == QS_SCALE_YOKED;
  if (cfg->num_tiles == 0) return QS_OK;
  if (!S0 || !codes || !scales || (yoked && !shadow)) return QS_ERR_INVALID_ARG;
  if (!aligned(S0, 16) || !aligned(codes, 32) || !aligned(scales, 16) || (yoked && !aligned(shadow, 32)))
    return QS_ERR_INVALID_ARG;
  const Sizes s = sizes_of(cfg);
  const Range w[3] = {range_of(codes, s.codes), range_of(scales, s.scales),
                      range_of(yoked ? shadow : nullptr, s.shadow)};
  const Range r[1] = {range_of(S0, static_cast<size_t>(cfg->num_tiles) * cfg->dv * cfg->dk * 4)};
  if (any_overlap(w, 3, r, 1)) return QS_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(cfg->num_tiles) * cfg->dv;
  uint8_t* c8 = static_cast<uint8_t*>(codes);
  float* sh = yoked ? shadow : nullptr;
  cudaError_t e;
  if (cfg->bits == 4)
    e = cfg->dk == 64 ? qs::launch_init<4, 64>(S0, c8, scales, sh, rows, cfg->group, stream)
                      : qs::launch_init<4, 128>(S0, c8, scales, sh, rows, cfg->group, stream);
  else
    e = cfg->dk == 64 ? qs::launch_init<8, 64>(S0, c8, scales, sh, rows, cfg->group, stream)
                      : qs::launch_init<8, 128>(S0, c8, scales, sh, rows, cfg->group, stream);
  return from_cuda(e);
}

qs_status qstate_decode_step(const qs_config* cfg, void* codes, float* scales, float* shadow,
                             const float* q, const float* k, const float* v, const float* alpha,
                             const float* beta, float* o, cudaStream_t stream) {
  qs_status st = check_config(cfg);
  if (st != QS_OK) return st;
  if (cfg->num_tiles == 0) return QS_OK;
  const bool yoked = cfg->policy == QS_SCALE_YOKED;
  const bool diag = cfg->decay == QS_DECAY_DIAGONAL;
  if (!codes || !scales || !k || !v || !alpha || !beta || (yoked && !shadow) || (o && !q))
    return QS_ERR_INVALID_ARG;
  if (!aligned(codes, 32) || !aligned(scales, 16) || !aligned(k, 16) || !aligned(v, 16) ||
      (q && !aligned(q, 16)) || (yoked && !aligned(shadow, 32)) || !aligned(alpha, diag ? 16 : 4) ||
      !aligned(beta, 4) || (o && !aligned(o, 4)))
    return QS_ERR_INVALID_ARG;
  const Sizes s = sizes_of(cfg);
  const Range w[4] = {range_of(codes, s.codes), range_of(scales, s.scales),
                      range_of(yoked ? shadow : nullptr, s.shadow), range_of(o, o ? s.vec_v : 0)};
  const Range r[5] = {range_of(q, q ? s.vec_k : 0), range_of(k, s.vec_k), range_of(v, s.vec_v),
                      range_of(alpha, s.alpha), range_of(beta, s.tile_scalars)};
  if (any_overlap(w, 4, r, 5)) return QS_ERR_INVALID_ARG;

  qs::StepParams p;
  p.codes = static_cast<uint8_t*>(codes);
  p.scales = scales;
  p.shadow = yoked ? shadow : nullptr;
  p.q = q;
  p.k = k;
  p.v = v;
  p.alpha = alpha;
  p.beta = beta;
  p.o = o;
  p.tiles = cfg->num_tiles;
  p.dv = cfg->dv;
  p.group = cfg->group;
  cudaError_t e;
  if (cfg->bits == 4)
    e = cfg->dk == 64 ? dispatch_step<4, 64>(cfg, p, stream) : dispatch_step<4, 128>(cfg, p, stream);
  else
    e = cfg->dk == 64 ? dispatch_step<8, 64>(cfg, p, stream) : dispatch_step<8, 128>(cfg, p, stream);
  return from_cuda(e);
}

qs_status qstate_fp32_decode_step(const qs_config* cfg, float* S, const float* q, const float* k,
                                  const float* v, const float* alpha, const float* beta, float* o,
                                  cudaStream_t stream) {
  if (cfg == nullptr) return QS_ERR_INVALID_ARG;
  // only the recurrence's fields matter here; check them through a quantized
  // configuration that is always valid for storage
  qs_config c = *cfg;
  c.bits = 8;
  c.group = 32;
  c.policy = QS_SCALE_PERSISTENT;
  c.rounding = QS_ROUND_NEAREST;
  qs_status st = check_config(&c);
  if (st != QS_OK) return st;
  if (c.num_tiles == 0) return QS_OK;
  const bool diag = c.decay == QS_DECAY_DIAGONAL;
  if (!S || !k || !v || !alpha || !beta || (o && !q)) return QS_ERR_INVALID_ARG;
  if (!aligned(S, 32) || !aligned(k, 16) || !aligned(v, 16) || (q && !aligned(q, 16)) ||
      !aligned(alpha, diag ? 16 : 4) || !aligned(beta, 4) || (o && !aligned(o, 4)))
    return QS_ERR_INVALID_ARG;
  const Sizes s = sizes_of(&c);
  const size_t state_bytes = static_cast<size_t>(c.num_tiles) * c.dv * c.dk * sizeof(float);
  const Range w[2] = {range_of(S, state_bytes), range_of(o, o ? s.vec_v : 0)};
  const Range r[5] = {range_of(q, q ? s.vec_k : 0), range_of(k, s.vec_k), range_of(v, s.vec_v),
                      range_of(alpha, s.alpha), range_of(beta, s.tile_scalars)};
  if (any_overlap(w, 2, r, 5)) return QS_ERR_INVALID_ARG;
  qs::StepParams p;
  std::memset(&p, 0, sizeof(p));
  p.shadow = S;
  p.q = q;
  p.k = k;
  p.v = v;
  p.alpha = alpha;
  p.beta = beta;
  p.o = o;
  p.tiles = c.num_tiles;
  p.dv = c.dv;
  p.group = c.group;
  const int sel = (c.dk == 128 ? 4 : 0) + (c.delta ? 2 : 0) + (diag ? 1 : 0);
  cudaError_t e;
  switch (sel) {
    case 0: e = qs::launch_fp32_step<64, false, false>(p, stream); break;
    case 1: e = qs::launch_fp32_step<64, false, true>(p, stream); break;
    case 2: e = qs::launch_fp32_step<64, true, false>(p, stream); break;
    case 3: e = qs::launch_fp32_step<64, true, true>(p, stream); break;
    case 4: e = qs::launch_fp32_step<128, false, false>(p, stream); break;
    case 5: e = qs::launch_fp32_step<128, false, true>(p, stream); break;
    case 6: e = qs::launch_fp32_step<128, true, false>(p, stream); break;
    default: e = qs::launch_fp32_step<128, true, true>(p, stream); break;
  }
  return from_cuda(e);
}

qs_status qstate_readout(const qs_config* cfg, const void* codes, const float* scales,
                         const float* q, float* o, cudaStream_t stream) {
  qs_status st = check_config(cfg);
  if (st != QS_OK) return st;
  if (cfg->num_tiles == 0) return QS_OK;
  if (!codes || !scales || !q || !o) return QS_ERR_INVALID_ARG;
  if (!aligned(codes, 32) || !aligned(scales, 16) || !aligned(q, 16) || !aligned(o, 4))
    return QS_ERR_INVALID_ARG;
  const Sizes s = sizes_of(cfg);
  const Range w[1] = {range_of(o, s.vec_v)};
  const Range r[3] = {range_of(codes, s.codes), range_of(scales, s.scales), range_of(q, s.vec_k)};
  if (any_overlap(w, 1, r, 3)) return QS_ERR_INVALID_ARG;
  qs::StepParams p;
  std::memset(&p, 0, sizeof(p));
  p.codes = const_cast<uint8_t*>(static_cast<const uint8_t*>(codes));
  p.scales = const_cast<float*>(scales);
  p.q = q;
  p.o = o;
  p.tiles = cfg->num_tiles;
  p.dv = cfg->dv;
  p.group = cfg->group;
  cudaError_t e;
  if (cfg->bits == 4)
    e = cfg->dk == 64 ? qs::launch_readout<4, 64>(p, stream) : qs::launch_readout<4, 128>(p, stream);
  else
    e = cfg->dk == 64 ? qs::launch_readout<8, 64>(p, stream) : qs::launch_readout<8, 128>(p, stream);
  return from_cuda(e);
}

qs_status qstate_lrb_query_sizes(const qs_config* cfg, int rank, size_t* decay_bytes,
                                 size_t* keys_bytes, size_t* coef_bytes) {
  qs_status st = check_config(cfg);
  if (st != QS_OK) return st;
  if (rank < 1 || rank > qs::kLrbMaxRank) return QS_ERR_UNSUPPORTED;
  const size_t T = static_cast<size_t>(cfg->num_tiles);
  if (decay_bytes) *decay_bytes = T * cfg->dk * sizeof(float);
  if (keys_bytes) *keys_bytes = T * rank * cfg->dk * sizeof(float);
  if (coef_bytes) *coef_bytes = T * cfg->dv * lrb_rpad(rank) * sizeof(float);
  return QS_OK;
}

qs_status qstate_lrb_decode_step(const qs_config* cfg, int rank, int slot, void* codes,
                                 float* scales, float* shadow, const float* A_in, float* A_out,
                                 const float* K_in, float* K_out, float* U, const float* q,
                                 const float* k, const float* v, const float* alpha,
                                 const float* beta, float* o, cudaStream_t stream) {
  qs_status st = check_config(cfg);
  if (st != QS_OK) return st;
  if (rank < 1 || rank > qs::kLrbMaxRank) return QS_ERR_UNSUPPORTED;
  if (slot < 0 || slot >= rank) return QS_ERR_INVALID_ARG;
  if (rank == 1)
    return qstate_decode_step(cfg, codes, scales, shadow, q, k, v, alpha, beta, o, stream);
  if (cfg->num_tiles == 0) return QS_OK;
  const bool merge = slot == rank - 1;
  const bool yoked = cfg->policy == QS_SCALE_YOKED;
  const bool diag = cfg->decay == QS_DECAY_DIAGONAL;
  if (!codes || !scales || !k || !v || !alpha || !beta || !U || (yoked && !shadow) || (o && !q))
    return QS_ERR_INVALID_ARG;
  if (slot > 0 && (!A_in || !K_in)) return QS_ERR_INVALID_ARG;
  if (!merge && (!A_out || !K_out)) return QS_ERR_INVALID_ARG;
  if (!aligned(codes, 32) || !aligned(scales, 16) || !aligned(k, 16) || !aligned(v, 16) ||
      (q && !aligned(q, 16)) || (yoked && !aligned(shadow, 32)) || !aligned(alpha, diag ? 16 : 4) ||
      !aligned(beta, 4) || (o && !aligned(o, 4)) || !aligned(U, 16) ||
      (A_in && slot > 0 && !aligned(A_in, 16)) || (K_in && slot > 0 && !aligned(K_in, 16)) ||
      (!merge && (!aligned(A_out, 16) || !aligned(K_out, 16))))
    return QS_ERR_INVALID_ARG;
  const Sizes s = sizes_of(cfg);
  size_t a_b = 0, k_b = 0, u_b = 0;
  qstate_lrb_query_sizes(cfg, rank, &a_b, &k_b, &u_b);
  const Range w[6] = {range_of(codes, s.codes), range_of(scales, s.scales),
                      range_of(yoked ? shadow : nullptr, s.shadow), range_of(o, o ? s.vec_v : 0),
                      range_of(U, u_b), range_of(merge ? nullptr : A_out, merge ? 0 : a_b)};
  const Range r[7] = {range_of(q, q ? s.vec_k : 0), range_of(k, s.vec_k), range_of(v, s.vec_v),
                      range_of(alpha, s.alpha), range_of(beta, s.tile_scalars),
                      range_of(slot > 0 ? A_in : nullptr, slot > 0 ? a_b : 0),
                      range_of(slot > 0 ? K_in : nullptr, slot > 0 ? k_b : 0)};
  if (any_overlap(w, 6, r, 7)) return QS_ERR_INVALID_ARG;
  if (!merge) {
    const Range w2[1] = {range_of(K_out, k_b)};
    const Range r2[2] = {range_of(slot > 0 ? K_in : nullptr, slot > 0 ? k_b : 0), w[0]};
    if (any_overlap(w2, 1, r2, 2)) return QS_ERR_INVALID_ARG;
    for (int i = 0; i < 6; ++i)
      if (overlap(w2[0], w[i])) return QS_ERR_INVALID_ARG;
  }
  qs::LrbParams p;
  std::memset(&p, 0, sizeof(p));
  p.codes = static_cast<uint8_t*>(codes);
  p.scales = scales;
  p.shadow = yoked ? shadow : nullptr;
  p.q = q;
  p.k = k;
  p.v = v;
  p.alpha = alpha;
  p.beta = beta;
  p.o = o;
  p.A_in = A_in;
  p.A_out = A_out;
  p.K_in = K_in;
  p.K_out = K_out;
  p.U = U;
  p.group = cfg->group;
  p.rank = rank;
  p.rpad = lrb_rpad(rank);
  p.slot = slot;
  cudaError_t e;
  if (cfg->bits == 4)
    e = cfg->dk == 64 ? dispatch_lrb<4, 64>(cfg, p, merge, stream) : dispatch_lrb<4, 128>(cfg, p, merge, stream);
  else
    e = cfg->dk == 64 ? dispatch_lrb<8, 64>(cfg, p, merge, stream) : dispatch_lrb<8, 128>(cfg, p, merge, stream);
  return from_cuda(e);
}

namespace {

// Validation shared by the two prefill paths; fills p and reports whether
// there is work to launch.
qs_status prefill_args(const qs_config* cfg, int length, float* S, const float* q, const float* k,
                       const float* v, const float* alpha, const float* beta, float* o, uintptr_t align,
                       bool allow_delta, qs_config* out, qs::PrefillParams* p, bool* work) {
  *work = false;
  if (cfg == nullptr) return QS_ERR_INVALID_ARG;
  qs_config c = *cfg;
  c.bits = 8;
  c.group = 32;
  c.policy = QS_SCALE_PERSISTENT;
  c.rounding = QS_ROUND_NEAREST;
  qs_status st = check_config(&c);
  if (st != QS_OK) return st;
  if ((c.delta != 0 && !allow_delta) || c.dv > 128) return QS_ERR_UNSUPPORTED;
  if (length < 0) return QS_ERR_INVALID_ARG;
  if (c.num_tiles == 0 || length == 0) return QS_OK;
  const bool diag = c.decay == QS_DECAY_DIAGONAL;
  if (!S || !q || !k || !v || !alpha || !beta) return QS_ERR_INVALID_ARG;
  if (!aligned(S, align) || !aligned(q, align) || !aligned(k, align) || !aligned(v, 4) ||
      !aligned(alpha, 4) || !aligned(beta, 4) || (o && !aligned(o, 4)))
    return QS_ERR_INVALID_ARG;
  const size_t T = static_cast<size_t>(c.num_tiles), L = static_cast<size_t>(length);
  const Range w[2] = {range_of(S, T * c.dv * c.dk * 4), range_of(o, o ? T * L * c.dv * 4 : 0)};
  const Range r[5] = {range_of(q, T * L * c.dk * 4), range_of(k, T * L * c.dk * 4),
                      range_of(v, T * L * c.dv * 4), range_of(alpha, T * L * (diag ? c.dk : 1) * 4),
                      range_of(beta, T * L * 4)};
  if (any_overlap(w, 2, r, 5)) return QS_ERR_INVALID_ARG;
  p->S = S;
  p->q = q;
  p->k = k;
  p->v = v;
  p->alpha = alpha;
  p->beta = beta;
  p->o = o;
  p->L = length;
  p->dv = c.dv;
  p->wait_probe = 0;
  *out = c;
  *work = true;
  return QS_OK;
}

}  // namespace

qs_status qstate_prefill(const qs_config* cfg, int length, float* S, const float* q,
                         const float* k, const float* v, const float* alpha, const float* beta,
                         float* o, cudaStream_t stream) {
  qs_config c;
  qs::PrefillParams p;
  bool work;
  const qs_status st = prefill_args(cfg, length, S, q, k, v, alpha, beta, o, 4, true, &c, &p, &work);
  if (st != QS_OK || !work) return st;
  const int sel = (c.dk == 128 ? 4 : 0) + (c.decay == QS_DECAY_DIAGONAL ? 2 : 0) + (c.delta ? 1 : 0);
  const int T = c.num_tiles;
  cudaError_t e;
  switch (sel) {
    case 0: e = qs::launch_prefill<64, false, false>(p, T, stream); break;
    case 1: e = qs::launch_prefill<64, false, true>(p, T, stream); break;
    case 2: e = qs::launch_prefill<64, true, false>(p, T, stream); break;
    case 3: e = qs::launch_prefill<64, true, true>(p, T, stream); break;
    case 4: e = qs::launch_prefill<128, false, false>(p, T, stream); break;
    case 5: e = qs::launch_prefill<128, false, true>(p, T, stream); break;
    case 6: e = qs::launch_prefill<128, true, false>(p, T, stream); break;
    default: e = qs::launch_prefill<128, true, true>(p, T, stream); break;
  }
  return from_cuda(e);
}

// Tensor-memory waits of the TF32 prefill that gave up (per device).
__device__ unsigned int qs_tc_timeouts = 0;

qs_status qstate_prefill_tf32(const qs_config* cfg, int length, float* S, const float* q,
                              const float* k, const float* v, const float* alpha, const float* beta,
                              float* o, cudaStream_t stream) {
  qs_config c;
  qs::PrefillParams p;
  bool work;
  // the delta rule runs on the FP32 path only
  const qs_status st = prefill_args(cfg, length, S, q, k, v, alpha, beta, o, 16, false, &c, &p, &work);
  if (st != QS_OK || !work) return st;
  unsigned int* timeouts = nullptr;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&timeouts), qs_tc_timeouts);
  if (e != cudaSuccess) return from_cuda(e);
  const bool diag = c.decay == QS_DECAY_DIAGONAL;
  const int T = c.num_tiles;
#define QS_TC(DK, M) (diag ? qs::launch_prefill_tc<DK, M, true>(p, T, timeouts, stream) \
                           : qs::launch_prefill_tc<DK, M, false>(p, T, timeouts, stream))
  if (c.dk == 64)
    e = c.dv <= 64 ? QS_TC(64, 64) : QS_TC(64, 128);
  else
    e = c.dv <= 64 ? QS_TC(128, 64) : QS_TC(128, 128);
#undef QS_TC
  return from_cuda(e);
}

qs_status qstate_prefill_tf32_wait_selfcheck(unsigned int polls, unsigned int* timed_out) {
  if (timed_out == nullptr || polls == 0 || polls > (1u << 20)) return QS_ERR_INVALID_ARG;
  unsigned int* timeouts = nullptr;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&timeouts), qs_tc_timeouts);
  unsigned int before = 0, after = 0;
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&before, qs_tc_timeouts, sizeof(unsigned int));
  if (e != cudaSuccess) return from_cuda(e);
  qs::PrefillParams p;
  std::memset(&p, 0, sizeof(p));
  p.L = 1;
  p.dv = 64;
  p.wait_probe = static_cast<int>(polls);
  e = qs::launch_prefill_tc<64, 64, false>(p, 1, timeouts, nullptr);
  if (e == cudaSuccess) e = cudaStreamSynchronize(nullptr);
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&after, qs_tc_timeouts, sizeof(unsigned int));
  if (e != cudaSuccess) return from_cuda(e);
  *timed_out = after - before;
  return QS_OK;
}

qs_status qstate_prefill_tf32_timeouts(unsigned int* count) {
  if (count == nullptr) return QS_ERR_INVALID_ARG;
  return from_cuda(cudaMemcpyFromSymbol(count, qs_tc_timeouts, sizeof(unsigned int)));
}

qs_status qstate_state_sq_norms(const qs_config* cfg, const void* codes, const float* scales,
                                double* out, cudaStream_t stream) {
  qs_status st = check_config(cfg);
  if (st != QS_OK) return st;
  if (cfg->num_tiles == 0) return QS_OK;
  if (!codes || !scales || !out) return QS_ERR_INVALID_ARG;
  if (!aligned(codes, 32) || !aligned(scales, 4) || !aligned(out, 8)) return QS_ERR_INVALID_ARG;
  const Sizes s = sizes_of(cfg);
  const Range w[1] = {range_of(out, static_cast<size_t>(cfg->num_tiles) * sizeof(double))};
  const Range r[2] = {range_of(codes, s.codes), range_of(scales, s.scales)};
  if (any_overlap(w, 1, r, 2)) return QS_ERR_INVALID_ARG;
  const uint8_t* c8 = static_cast<const uint8_t*>(codes);
  const dim3 grid(static_cast<unsigned>(cfg->num_tiles)), block(qs::kNormThreads);
  if (cfg->bits == 4) {
    if (cfg->dk == 64)
      qs::state_sq_norm_kernel<4, 64><<<grid, block, 0, stream>>>(c8, scales, out, cfg->dv, cfg->group);
    else
      qs::state_sq_norm_kernel<4, 128><<<grid, block, 0, stream>>>(c8, scales, out, cfg->dv, cfg->group);
  } else {
    if (cfg->dk == 64)
      qs::state_sq_norm_kernel<8, 64><<<grid, block, 0, stream>>>(c8, scales, out, cfg->dv, cfg->group);
    else
      qs::state_sq_norm_kernel<8, 128><<<grid, block, 0, stream>>>(c8, scales, out, cfg->dv, cfg->group);
  }
  return from_cuda(cudaGetLastError());
}

qs_status qstate_fp32_sq_norms(const qs_config* cfg, const float* S, double* out,
                               cudaStream_t stream) {
  if (cfg == nullptr) return QS_ERR_INVALID_ARG;
  qs_config c = *cfg;
  c.bits = 8;
  c.group = 32;
  c.policy = QS_SCALE_PERSISTENT;
  c.rounding = QS_ROUND_NEAREST;
  qs_status st = check_config(&c);
  if (st != QS_OK) return st;
  if (c.num_tiles == 0) return QS_OK;
  if (!S || !out) return QS_ERR_INVALID_ARG;
  if (!aligned(S, 16) || !aligned(out, 8)) return QS_ERR_INVALID_ARG;
  const size_t elems = static_cast<size_t>(c.dv) * c.dk;
  const Range w[1] = {range_of(out, static_cast<size_t>(c.num_tiles) * sizeof(double))};
  const Range r[1] = {range_of(S, static_cast<size_t>(c.num_tiles) * elems * sizeof(float))};
  if (any_overlap(w, 1, r, 1)) return QS_ERR_INVALID_ARG;
  qs::fp32_sq_norm_kernel<<<static_cast<unsigned>(c.num_tiles), qs::kNormThreads, 0, stream>>>(
      S, out, static_cast<long long>(elems));
  return from_cuda(cudaGetLastError());
}

}  // extern "C"
