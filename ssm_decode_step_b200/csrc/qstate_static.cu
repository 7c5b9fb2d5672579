// qstate_decode_step_host_static (include/qstate.h): one decode step whose
// inputs come from host memory and whose readouts go back there, staged on
// the device through a fixed array that the library owns, so that the call
// allocates no memory at all.
//
// Who needs it: a caller that may not allocate device memory on its own,
// for instance an engine whose memory manager owns the whole device budget
// (a cudaMalloc outside it can fail or fragment that budget), or a serving
// loop that must not pay cudaMalloc's device-wide synchronization on the
// decode path.  The host-buffer pipeline (qstate_pipeline_*) stages through
// buffers it allocates at creation; this entry point stages through the
// array below instead.
//
// The array is a file-scope __device__ variable: every GPU that loads this
// library holds its kQsStaticStageBytes until the process exits.  In host
// code its name is only a host-side stand-in for the symbol, not a device
// address, so the device address is looked up once per device with
// cudaGetSymbolAddress (with that device current) and passed to the
// kernels; handing the host-side name to a kernel would read the wrong
// memory or fault.
#include <cstdint>
#include <mutex>

#include "../../include/qstate.h"

namespace {

constexpr size_t kQsStaticStageBytes = QS_STATIC_STAGE_BYTES;
constexpr int kMaxDevices = 64;

// The staging area: one step's packed inputs (q | k | v | alpha | beta),
// then its readouts.  Every byte a call reads from it was written by the
// same call first, so nothing in it needs to start at zero.
static __device__ __align__(256) unsigned char qs_static_stage[kQsStaticStageBytes];

std::mutex g_mu;
void* g_stage[kMaxDevices] = {};

// The device address of the staging array on the current device, looked up
// on the first call for that device.
cudaError_t stage_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_stage[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, qs_static_stage);
    if (e != cudaSuccess) return e;
    g_stage[dev] = p;
  }
  *out = g_stage[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

QS_API qs_status qstate_decode_step_host_static(const qs_config* cfg, void* codes, float* scales,
                                                float* shadow, const void* host_in, float* host_out,
                                                cudaStream_t stream) {
  if (cfg == nullptr || host_in == nullptr) return QS_ERR_INVALID_ARG;
  size_t in_bytes = 0, out_bytes = 0;
  qs_status st = qstate_pipeline_query_sizes(cfg, 1, &in_bytes, &out_bytes);
  if (st != QS_OK) return st;
  if (cfg->num_tiles == 0) return QS_OK;
  const size_t need = in_bytes + (host_out ? out_bytes : 0);
  if (need > kQsStaticStageBytes) return QS_ERR_UNSUPPORTED;
  void* base = nullptr;
  cudaError_t e = stage_address(&base);
  if (e != cudaSuccess) return QS_ERR_CUDA;
  unsigned char* in = static_cast<unsigned char*>(base);
  // the packed layout of qstate_pipeline_query_sizes: q | k | v | alpha | beta
  const size_t T = static_cast<size_t>(cfg->num_tiles);
  const float* q = reinterpret_cast<const float*>(in);
  const float* k = q + T * cfg->dk;
  const float* v = k + T * cfg->dk;
  const float* alpha = v + T * cfg->dv;
  const float* beta = alpha + (cfg->decay == QS_DECAY_DIAGONAL ? T * cfg->dk : T);
  float* o = host_out ? reinterpret_cast<float*>(in + in_bytes) : nullptr;
  if ((e = cudaMemcpyAsync(in, host_in, in_bytes, cudaMemcpyHostToDevice, stream)) != cudaSuccess)
    return QS_ERR_CUDA;
  st = qstate_decode_step(cfg, codes, scales, shadow, o ? q : nullptr, k, v, alpha, beta, o, stream);
  if (st != QS_OK) return st;
  if (host_out &&
      (e = cudaMemcpyAsync(host_out, o, out_bytes, cudaMemcpyDeviceToHost, stream)) != cudaSuccess)
    return QS_ERR_CUDA;
  return QS_OK;
}

}  // extern "C"
