// Host-buffer decode pipeline (qstate_pipeline_* of include/qstate.h): the
// serving loop around qstate_decode_step when a token's inputs arrive in
// host memory and its readouts go back there.
//
// Per step t (buffer b = t mod depth):
//   host   wait for the output copy of step t - depth (it last used buffer b)
//   copy-in stream    inputs  host -> d_in[b];        record up[b]
//   caller's stream   wait up[b]; one decode step per family, reading d_in[b]
//                     and writing readouts to d_out[b]; record done[b]
//   copy-out stream   wait done[b]; readouts d_out[b] -> host; record down[b]
// so the copies of one step overlap the state updates of its neighbours,
// the state updates stay in call order on the caller's stream, and the host
// runs at most `depth` steps ahead of the copies.  Everything here is host
// code; the arithmetic is in the step kernels behind qstate_decode_step.
#include <cstdint>
#include <cstring>
#include <new>

#include "../../include/qstate.h"

namespace {

constexpr int kMaxFamilies = 8;
constexpr int kMinDepth = 2, kMaxDepth = 8;

struct Layout {
  size_t q, k, v, alpha, beta, in_bytes, out_family;
};

// Byte offsets of the packed host input of one step (q | k | v | alpha |
// beta) and the bytes of one family's readout.  With dk in {64, 128} and dv
// a multiple of 16 every part starts on the boundary its kernel argument
// needs (16 bytes for q, k, v and diagonal alpha, 4 for the rest).
Layout layout_of(const qs_config& c) {
  const size_t T = static_cast<size_t>(c.num_tiles);
  Layout L;
  size_t off = 0;
  L.q = off;     off += T * c.dk * sizeof(float);
  L.k = off;     off += T * c.dk * sizeof(float);
  L.v = off;     off += T * c.dv * sizeof(float);
  L.alpha = off; off += (c.decay == QS_DECAY_DIAGONAL ? T * c.dk : T) * sizeof(float);
  L.beta = off;  off += T * sizeof(float);
  L.in_bytes = off;
  L.out_family = T * c.dv * sizeof(float);
  return L;
}

bool same_recurrence(const qs_config& a, const qs_config& b) {
  return a.num_tiles == b.num_tiles && a.dk == b.dk && a.dv == b.dv && a.delta == b.delta &&
         a.decay == b.decay;
}

qs_status check_families(int n, const qs_config* cfgs) {
  if (cfgs == nullptr || n < 1 || n > kMaxFamilies) return QS_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    const qs_status st = qstate_query_sizes(&cfgs[i], nullptr, nullptr, nullptr);
    if (st != QS_OK) return st;
    if (!same_recurrence(cfgs[0], cfgs[i])) return QS_ERR_INVALID_ARG;
  }
  return QS_OK;
}

qs_status from_cuda(cudaError_t e) { return e == cudaSuccess ? QS_OK : QS_ERR_CUDA; }

}  // namespace

struct qs_pipeline {
  int n = 0, depth = 0, device = 0;
  qs_config cfg[kMaxFamilies];
  Layout L;
  unsigned char* d_in[kMaxDepth] = {};
  unsigned char* d_out[kMaxDepth] = {};
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t up[kMaxDepth] = {}, done[kMaxDepth] = {}, down[kMaxDepth] = {};
  cudaEvent_t mark = nullptr;
  long long issued = 0;

  // Frees whatever was created; safe on a partly built pipeline.
  void release() {
    for (int b = 0; b < kMaxDepth; ++b) {
      if (d_in[b]) cudaFree(d_in[b]);
      if (d_out[b]) cudaFree(d_out[b]);
      if (up[b]) cudaEventDestroy(up[b]);
      if (done[b]) cudaEventDestroy(done[b]);
      if (down[b]) cudaEventDestroy(down[b]);
      d_in[b] = d_out[b] = nullptr;
      up[b] = done[b] = down[b] = nullptr;
    }
    if (mark) cudaEventDestroy(mark);
    if (s_in) cudaStreamDestroy(s_in);
    if (s_out) cudaStreamDestroy(s_out);
    mark = nullptr;
    s_in = s_out = nullptr;
  }

  cudaError_t build() {
    cudaError_t e = cudaGetDevice(&device);
    if (e != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&mark, cudaEventDisableTiming)) != cudaSuccess) return e;
    for (int b = 0; b < depth; ++b) {
      if ((e = cudaMalloc(&d_in[b], L.in_bytes)) != cudaSuccess) return e;
      if ((e = cudaMalloc(&d_out[b], n * L.out_family)) != cudaSuccess) return e;
      if ((e = cudaEventCreateWithFlags(&up[b], cudaEventDisableTiming)) != cudaSuccess) return e;
      if ((e = cudaEventCreateWithFlags(&done[b], cudaEventDisableTiming)) != cudaSuccess) return e;
      if ((e = cudaEventCreateWithFlags(&down[b], cudaEventDisableTiming)) != cudaSuccess) return e;
    }
    return cudaSuccess;
  }

  bool on_own_device() const {
    int dev = -1;
    return cudaGetDevice(&dev) == cudaSuccess && dev == device;
  }
};

extern "C" {

qs_status qstate_pipeline_query_sizes(const qs_config* cfg, int n, size_t* in_bytes,
                                      size_t* out_bytes) {
  if (cfg == nullptr || n < 1 || n > kMaxFamilies) return QS_ERR_INVALID_ARG;
  const qs_status st = qstate_query_sizes(cfg, nullptr, nullptr, nullptr);
  if (st != QS_OK) return st;
  const Layout L = layout_of(*cfg);
  if (in_bytes) *in_bytes = L.in_bytes;
  if (out_bytes) *out_bytes = n * L.out_family;
  return QS_OK;
}

qs_status qstate_pipeline_create(int n, const qs_config* cfgs, int depth, qs_pipeline** out) {
  if (out == nullptr) return QS_ERR_INVALID_ARG;
  *out = nullptr;
  const qs_status st = check_families(n, cfgs);
  if (st != QS_OK) return st;
  if (depth < kMinDepth || depth > kMaxDepth) return QS_ERR_INVALID_ARG;
  qs_pipeline* pl = new (std::nothrow) qs_pipeline;
  if (pl == nullptr) return QS_ERR_CUDA;
  pl->n = n;
  pl->depth = depth;
  std::memcpy(pl->cfg, cfgs, n * sizeof(qs_config));
  pl->L = layout_of(cfgs[0]);
  const cudaError_t e = pl->build();
  if (e != cudaSuccess) {
    pl->release();
    delete pl;
    return QS_ERR_CUDA;
  }
  *out = pl;
  return QS_OK;
}

qs_status qstate_pipeline_step(qs_pipeline* pl, void* const* codes, float* const* scales,
                               float* const* shadow, const void* host_in, void* host_out,
                               cudaStream_t stream) {
  if (pl == nullptr || codes == nullptr || scales == nullptr || host_in == nullptr)
    return QS_ERR_INVALID_ARG;
  for (int i = 0; i < pl->n; ++i) {
    if (codes[i] == nullptr || scales[i] == nullptr) return QS_ERR_INVALID_ARG;
    if (pl->cfg[i].policy == QS_SCALE_YOKED && (shadow == nullptr || shadow[i] == nullptr))
      return QS_ERR_INVALID_ARG;
  }
  if (!pl->on_own_device()) return QS_ERR_INVALID_ARG;
  const int b = static_cast<int>(pl->issued % pl->depth);
  cudaError_t e;
  // the step that last used buffer b has finished with it, copies included
  if (pl->issued >= pl->depth && (e = cudaEventSynchronize(pl->down[b])) != cudaSuccess)
    return from_cuda(e);
  const Layout& L = pl->L;
  unsigned char* in = pl->d_in[b];
  if ((e = cudaMemcpyAsync(in, host_in, L.in_bytes, cudaMemcpyHostToDevice, pl->s_in)) != cudaSuccess ||
      (e = cudaEventRecord(pl->up[b], pl->s_in)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(stream, pl->up[b], 0)) != cudaSuccess)
    return from_cuda(e);
  const float* q = reinterpret_cast<const float*>(in + L.q);
  const float* k = reinterpret_cast<const float*>(in + L.k);
  const float* v = reinterpret_cast<const float*>(in + L.v);
  const float* alpha = reinterpret_cast<const float*>(in + L.alpha);
  const float* beta = reinterpret_cast<const float*>(in + L.beta);
  for (int i = 0; i < pl->n; ++i) {
    float* o = host_out ? reinterpret_cast<float*>(pl->d_out[b] + i * L.out_family) : nullptr;
    const qs_status st = qstate_decode_step(&pl->cfg[i], codes[i], scales[i], shadow ? shadow[i] : nullptr,
                                            o ? q : nullptr, k, v, alpha, beta, o, stream);
    if (st != QS_OK) return st;
  }
  if ((e = cudaEventRecord(pl->done[b], stream)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(pl->s_out, pl->done[b], 0)) != cudaSuccess)
    return from_cuda(e);
  if (host_out &&
      (e = cudaMemcpyAsync(host_out, pl->d_out[b], pl->n * L.out_family, cudaMemcpyDeviceToHost,
                           pl->s_out)) != cudaSuccess)
    return from_cuda(e);
  if ((e = cudaEventRecord(pl->down[b], pl->s_out)) != cudaSuccess) return from_cuda(e);
  ++pl->issued;
  return QS_OK;
}

qs_status qstate_pipeline_wait_stream(qs_pipeline* pl, cudaStream_t stream) {
  if (pl == nullptr) return QS_ERR_INVALID_ARG;
  if (!pl->on_own_device()) return QS_ERR_INVALID_ARG;
  cudaError_t e;
  if ((e = cudaEventRecord(pl->mark, stream)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(pl->s_in, pl->mark, 0)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(pl->s_out, pl->mark, 0)) != cudaSuccess)
    return from_cuda(e);
  return QS_OK;
}

qs_status qstate_pipeline_join(qs_pipeline* pl, cudaStream_t stream) {
  if (pl == nullptr) return QS_ERR_INVALID_ARG;
  if (!pl->on_own_device()) return QS_ERR_INVALID_ARG;
  if (pl->issued == 0) return QS_OK;
  // the last step's output copy follows every earlier copy on its stream,
  // and its input copy precedes its state updates
  const int b = static_cast<int>((pl->issued - 1) % pl->depth);
  return from_cuda(cudaStreamWaitEvent(stream, pl->down[b], 0));
}

qs_status qstate_pipeline_sync(qs_pipeline* pl) {
  if (pl == nullptr) return QS_ERR_INVALID_ARG;
  if (pl->issued == 0) return QS_OK;
  const int b = static_cast<int>((pl->issued - 1) % pl->depth);
  return from_cuda(cudaEventSynchronize(pl->down[b]));
}

qs_status qstate_pipeline_destroy(qs_pipeline* pl) {
  if (pl == nullptr) return QS_OK;
  const qs_status st = qstate_pipeline_sync(pl);
  pl->release();
  delete pl;
  return st;
}

}  // extern "C"
