// Definitions of the launchers declared in qstate_launch.h.
#pragma once

#include <cstdlib>
#include <mutex>

#include "qstate_launch.h"

namespace qs {

// Ring depth of the step kernel (row blocks per lane).
template <int POLICY>
constexpr int step_depth() { return POLICY == 2 ? QS_DEPTH_YOKED : QS_DEPTH; }

// Allow the kernel the device's full opt-in shared memory (once per kernel).
template <typename K>
static cudaError_t allow_smem(K kernel, std::once_flag& flag) {
  cudaError_t err = cudaSuccess;
  std::call_once(flag, [&] {
    int dev = 0, optin = 0;
    err = cudaGetDevice(&dev);
    if (err == cudaSuccess) err = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (err == cudaSuccess)
      err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
  });
  return err;
}

// Programmatic dependent launch for the streaming kernels (step, Low-Rank
// Bypass step, readout, FP32-state step): each may be scheduled while the
// kernel before it in the stream finishes, and waits for it in
// grid_dep_wait() before touching global memory.  QSTATE_PDL=0 in the
// environment launches them plainly.
static bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("QSTATE_PDL");
    return !(e && e[0] == '0' && e[1] == '\0');
  }();
  return on;
}

template <typename K, typename P>
static cudaError_t launch_dependent(K kernel, long long grid, int threads, size_t smem,
                                    cudaStream_t stream, const P& p) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

// Resident CTAs per SM of `kernel` at `threads` threads and `smem` bytes of
// dynamic shared memory on the current device, cached per (kernel, device,
// threads, smem): the occupancy query costs more host time than a launch.
template <typename K>
static cudaError_t resident_ctas(K kernel, int threads, size_t smem, int* per_sm) {
  struct Entry {
    const void* fn;
    int dev, threads, n;
    size_t smem;
  };
  static std::mutex mu;
  static Entry cache[64];
  static int used = 0;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const void* fn = reinterpret_cast<const void*>(kernel);
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i) {
      const Entry& e = cache[i];
      if (e.fn == fn && e.dev == dev && e.threads == threads && e.smem == smem) {
        *per_sm = e.n;
        return cudaSuccess;
      }
    }
  }
  int n = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem);
  if (err != cudaSuccess) return err;
  std::lock_guard<std::mutex> lock(mu);
  if (used < 64) cache[used++] = Entry{fn, dev, threads, n, smem};
  *per_sm = n;
  return cudaSuccess;
}

template <typename K>
static cudaError_t launch_persistent(K kernel, size_t smem, const StepParams& p,
                                     cudaStream_t stream) {
  int per_sm = 0;
  cudaError_t err = resident_ctas(kernel, kThreads, smem, &per_sm);
  if (err != cudaSuccess) return err;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const long long units = static_cast<long long>(p.tiles) * p.units_per_tile;
  long long grid = static_cast<long long>(per_sm) * device_sm_count();
  if (grid > units) grid = units;
  StepParams q = p;
  q.grid_tiles = static_cast<int>(grid / p.units_per_tile);
  q.grid_part = static_cast<int>(grid % p.units_per_tile);
  return launch_dependent(kernel, grid, kThreads, smem, stream, q);
}

// Launch a one-warp-per-range kernel (step, Low-Rank Bypass step, readout):
// as many CTAs as stay resident on all SMs, at most one warp per row block.
template <typename K, typename P>
static cudaError_t launch_warps(K kernel, const P& p, size_t smem, cudaStream_t stream) {
  int per_sm = 0;
  cudaError_t err = resident_ctas(kernel, kStepThreads, smem, &per_sm);
  if (err != cudaSuccess) return err;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  long long grid = static_cast<long long>(per_sm) * device_sm_count();
  const long long need = (static_cast<long long>(p.nblocks) + kStepWarps - 1) / kStepWarps;
  if (grid > need) grid = need;
  return launch_dependent(kernel, grid, kStepThreads, smem, stream, p);
}

// The decode step: the streamed kernel for the dynamic and persistent
// policies, the shared-memory ring kernel for the yoked policy (whose FP32
// shadow is too large to stream through registers).
template <int BITS, int DK, int POLICY, bool BDR, bool DELTA, bool DIAG>
cudaError_t launch_step(const StepParams& p0, cudaStream_t stream) {
  constexpr int RW = 32 / (DK / 32);  // rows per row block
  if constexpr (POLICY != 2) {
    auto kernel = stream_step_kernel<BITS, DK, POLICY, BDR, DELTA, DIAG>;
    static std::once_flag flag;
    cudaError_t err = allow_smem(kernel, flag);
    if (err != cudaSuccess) return err;
    StreamParams p;
    p.codes = p0.codes;
    p.scales = p0.scales;
    p.q = p0.q;
    p.k = p0.k;
    p.v = p0.v;
    p.alpha = p0.alpha;
    p.beta = p0.beta;
    p.o = p0.o;
    p.bpt = p0.dv / RW;
    p.nblocks = p0.tiles * p.bpt;  // < 2^31 (checked by the caller)
    p.group = p0.group;
    p.two23 = 0x4B000000u;
    const StreamLayout L(DK, DIAG, BDR && POLICY == 0);
    int per_sm = 0;
    err = resident_ctas(kernel, 32, static_cast<size_t>(L.bytes()), &per_sm);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    long long grid = static_cast<long long>(per_sm) * device_sm_count();
    if (grid > p.nblocks) grid = p.nblocks;
    return launch_dependent(kernel, grid, 32, static_cast<size_t>(L.bytes()), stream, p);
  } else {
    constexpr int D = step_depth<POLICY>();
    constexpr int WARPS = kStepWarps;
    auto kernel = step_kernel<BITS, DK, POLICY, BDR, DELTA, DIAG, D>;
    static std::once_flag flag;
    cudaError_t err = allow_smem(kernel, flag);
    if (err != cudaSuccess) return err;
    WarpStepParams p;
    p.codes = p0.codes;
    p.scales = p0.scales;
    p.shadow = p0.shadow;
    p.q = p0.q;
    p.k = p0.k;
    p.v = p0.v;
    p.alpha = p0.alpha;
    p.beta = p0.beta;
    p.o = p0.o;
    p.bpt = p0.dv / RW;
    p.nblocks = p0.tiles * p.bpt;  // < 2^31 (checked by the caller)
    p.group = p0.group;
    // tile-vector slots: every tile that D consecutive row blocks can touch
    p.ntv = (D - 1 + p.bpt - 1) / p.bpt + 1;
    const WarpLayout L(BITS, DK, DIAG, BDR, true);
    p.warp_bytes = L.bytes(D, p.ntv);
    return launch_warps(kernel, p, static_cast<size_t>(p.warp_bytes) * WARPS, stream);
  }
}

// The Low-Rank Bypass step: the streamed bypass kernel for the steps that
// keep the stored state under the dynamic and persistent policies, the ring
// kernel for the merge and for the yoked policy.
template <int BITS, int DK, int POLICY, bool BDR, bool DELTA, bool DIAG, bool MERGE>
cudaError_t launch_lrb(const LrbParams& p0, int tiles, int dv, cudaStream_t stream) {
  constexpr int D = 2;
  constexpr int RW = 32 / (DK / 32);
  constexpr int WARPS = kStepWarps;
  if constexpr (POLICY != 2 && !MERGE) {
    // coefficient registers for ranks up to 8, or up to 16
    const bool small = p0.rpad <= 8;
    auto kernel = small ? lrb_bypass_kernel<BITS, DK, DELTA, DIAG, 2> : lrb_bypass_kernel<BITS, DK, DELTA, DIAG, 4>;
    static std::once_flag flag_small, flag_large;
    cudaError_t err = allow_smem(kernel, small ? flag_small : flag_large);
    if (err != cudaSuccess) return err;
    LrbParams p = p0;
    p.bpt = dv / RW;
    p.nblocks = tiles * p.bpt;  // < 2^31 (checked by the caller)
    p.two23 = 0x4B000000u;
    const BypassLayout L(DK, DIAG, p.rank);
    int per_sm = 0;
    err = resident_ctas(kernel, 32, static_cast<size_t>(L.bytes()), &per_sm);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    long long grid = static_cast<long long>(per_sm) * device_sm_count();
    if (grid > p.nblocks) grid = p.nblocks;
    return launch_dependent(kernel, grid, 32, static_cast<size_t>(L.bytes()), stream, p);
  }
  auto kernel = lrb_step_kernel<BITS, DK, POLICY, BDR, DELTA, DIAG, MERGE, D>;
  static std::once_flag flag;
  cudaError_t err = allow_smem(kernel, flag);
  if (err != cudaSuccess) return err;
  LrbParams p = p0;
  p.bpt = dv / RW;
  p.nblocks = tiles * p.bpt;
  p.ntv = (D - 1 + p.bpt - 1) / p.bpt + 1;
  const LrbLayout L(BITS, DK, DIAG, POLICY == 2, MERGE, p.rank, p.rpad);
  p.warp_bytes = L.bytes(D, p.ntv);
  return launch_warps(kernel, p, static_cast<size_t>(p.warp_bytes) * WARPS, stream);
}

template <int BITS, int DK>
cudaError_t launch_readout(const StepParams& p0, cudaStream_t stream) {
  constexpr int D = QS_DEPTH;
  constexpr int RW = 32 / (DK / 32);
  auto kernel = readout_kernel<BITS, DK, D>;
  static std::once_flag flag;
  cudaError_t err = allow_smem(kernel, flag);
  if (err != cudaSuccess) return err;
  WarpStepParams p{};
  p.codes = p0.codes;
  p.scales = p0.scales;
  p.q = p0.q;
  p.o = p0.o;
  p.bpt = p0.dv / RW;
  p.nblocks = p0.tiles * p.bpt;
  p.group = p0.group;
  p.ntv = (D - 1 + p.bpt - 1) / p.bpt + 1;
  const WarpLayout L(BITS, DK, false, false, false);
  p.warp_bytes = L.bytes(D, p.ntv);
  return launch_warps(kernel, p, static_cast<size_t>(p.warp_bytes) * kStepWarps, stream);
}

template <int BITS, int DK>
cudaError_t launch_init(const float* S0, uint8_t* codes, float* scales, float* shadow,
                        long long rows, int group, cudaStream_t stream) {
  const long long threads = rows * (DK / 32);
  const long long blocks = (threads + 255) / 256;
  init_kernel<BITS, DK><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(S0, codes, scales, shadow,
                                                                         rows, group);
  return cudaGetLastError();
}

#define QS_INSTANTIATE_STEP(B, D, P, R, DE, DI) \
  template cudaError_t launch_step<B, D, P, R, DE, DI>(const StepParams&, cudaStream_t);

#define QS_INSTANTIATE_ALL(B, D)                                                      \
  QS_INSTANTIATE_STEP(B, D, 0, false, false, false) QS_INSTANTIATE_STEP(B, D, 0, false, false, true) \
  QS_INSTANTIATE_STEP(B, D, 0, false, true, false)  QS_INSTANTIATE_STEP(B, D, 0, false, true, true)  \
  QS_INSTANTIATE_STEP(B, D, 0, true, false, false)  QS_INSTANTIATE_STEP(B, D, 0, true, false, true)  \
  QS_INSTANTIATE_STEP(B, D, 0, true, true, false)   QS_INSTANTIATE_STEP(B, D, 0, true, true, true)   \
  QS_INSTANTIATE_STEP(B, D, 1, false, false, false) QS_INSTANTIATE_STEP(B, D, 1, false, false, true) \
  QS_INSTANTIATE_STEP(B, D, 1, false, true, false)  QS_INSTANTIATE_STEP(B, D, 1, false, true, true)  \
  QS_INSTANTIATE_STEP(B, D, 1, true, false, false)  QS_INSTANTIATE_STEP(B, D, 1, true, false, true)  \
  QS_INSTANTIATE_STEP(B, D, 1, true, true, false)   QS_INSTANTIATE_STEP(B, D, 1, true, true, true)   \
  QS_INSTANTIATE_STEP(B, D, 2, false, false, false) QS_INSTANTIATE_STEP(B, D, 2, false, false, true) \
  QS_INSTANTIATE_STEP(B, D, 2, false, true, false)  QS_INSTANTIATE_STEP(B, D, 2, false, true, true)  \
  QS_INSTANTIATE_STEP(B, D, 2, true, false, false)  QS_INSTANTIATE_STEP(B, D, 2, true, false, true)  \
  QS_INSTANTIATE_STEP(B, D, 2, true, true, false)   QS_INSTANTIATE_STEP(B, D, 2, true, true, true)   \
  template cudaError_t launch_readout<B, D>(const StepParams&, cudaStream_t);        \
  template cudaError_t launch_init<B, D>(const float*, uint8_t*, float*, float*, long long, int, \
                                         cudaStream_t);

#define QS_INSTANTIATE_LRB1(B, D, P, R, DE, DI, M) \
  template cudaError_t launch_lrb<B, D, P, R, DE, DI, M>(const LrbParams&, int, int, cudaStream_t);

// bypass steps requantize nothing, so only the yoked shadow distinguishes
// the policies there (0 stands for dynamic and persistent)
#define QS_INSTANTIATE_LRB(B, D)                                                                \
  QS_INSTANTIATE_LRB1(B, D, 0, false, false, false, false) QS_INSTANTIATE_LRB1(B, D, 0, false, false, true, false) \
  QS_INSTANTIATE_LRB1(B, D, 0, false, true, false, false)  QS_INSTANTIATE_LRB1(B, D, 0, false, true, true, false)  \
  QS_INSTANTIATE_LRB1(B, D, 2, false, false, false, false) QS_INSTANTIATE_LRB1(B, D, 2, false, false, true, false) \
  QS_INSTANTIATE_LRB1(B, D, 2, false, true, false, false)  QS_INSTANTIATE_LRB1(B, D, 2, false, true, true, false)  \
  QS_INSTANTIATE_LRB1(B, D, 0, false, false, false, true) QS_INSTANTIATE_LRB1(B, D, 0, false, false, true, true) \
  QS_INSTANTIATE_LRB1(B, D, 0, false, true, false, true)  QS_INSTANTIATE_LRB1(B, D, 0, false, true, true, true)  \
  QS_INSTANTIATE_LRB1(B, D, 0, true, false, false, true)  QS_INSTANTIATE_LRB1(B, D, 0, true, false, true, true)  \
  QS_INSTANTIATE_LRB1(B, D, 0, true, true, false, true)   QS_INSTANTIATE_LRB1(B, D, 0, true, true, true, true)   \
  QS_INSTANTIATE_LRB1(B, D, 1, false, false, false, true) QS_INSTANTIATE_LRB1(B, D, 1, false, false, true, true) \
  QS_INSTANTIATE_LRB1(B, D, 1, false, true, false, true)  QS_INSTANTIATE_LRB1(B, D, 1, false, true, true, true)  \
  QS_INSTANTIATE_LRB1(B, D, 1, true, false, false, true)  QS_INSTANTIATE_LRB1(B, D, 1, true, false, true, true)  \
  QS_INSTANTIATE_LRB1(B, D, 1, true, true, false, true)   QS_INSTANTIATE_LRB1(B, D, 1, true, true, true, true)   \
  QS_INSTANTIATE_LRB1(B, D, 2, false, false, false, true) QS_INSTANTIATE_LRB1(B, D, 2, false, false, true, true) \
  QS_INSTANTIATE_LRB1(B, D, 2, false, true, false, true)  QS_INSTANTIATE_LRB1(B, D, 2, false, true, true, true)  \
  QS_INSTANTIATE_LRB1(B, D, 2, true, false, false, true)  QS_INSTANTIATE_LRB1(B, D, 2, true, false, true, true)  \
  QS_INSTANTIATE_LRB1(B, D, 2, true, true, false, true)   QS_INSTANTIATE_LRB1(B, D, 2, true, true, true, true)

}  // namespace qs
