// Definitions of the launchers declared in qstate_launch_prefill.h.
#pragma once

#include "qstate_launch_impl.cuh"
#include "qstate_launch_prefill.h"

namespace qs {

#ifndef QS_PREFILL_WIDE
#define QS_PREFILL_WIDE 1
#endif

template <int DK, bool DIAG, bool DELTA>
cudaError_t launch_prefill(const PrefillParams& p, int tiles, cudaStream_t stream) {
  auto narrow = prefill_kernel<DK, DIAG, DELTA, kPrefillThreads>;
  auto wide = prefill_kernel<DK, DIAG, DELTA, kPrefillThreadsWide>;
  static std::once_flag f1, f2;
  cudaError_t err = allow_smem(narrow, f1);
  if (err == cudaSuccess) err = allow_smem(wide, f2);
  if (err != cudaSuccess) return err;
  const PrefillLayout L(DK, p.dv, DIAG, DELTA);
  const size_t smem = static_cast<size_t>(L.total) * sizeof(float);
  // 16 warps in one CTA where two CTAs of 8 warps do not fit on an SM
  int per_sm = 0;
  err = resident_ctas(narrow, kPrefillThreads, smem, &per_sm);
  if (err != cudaSuccess) return err;
  if (QS_PREFILL_WIDE && per_sm < 2)
    wide<<<tiles, kPrefillThreadsWide, smem, stream>>>(p);
  else
    narrow<<<tiles, kPrefillThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

template <int DK, int MDV, bool DIAG>
cudaError_t launch_prefill_tc(const PrefillParams& p, int tiles, unsigned int* timeouts,
                              cudaStream_t stream) {
  auto kernel = prefill_tc_kernel<DK, MDV, DIAG>;
  static std::once_flag flag;
  cudaError_t err = allow_smem(kernel, flag);
  if (err != cudaSuccess) return err;
  const size_t smem = static_cast<size_t>(TcLayout(DK, DIAG).bytes());
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kTcThreads, smem);
  if (err != cudaSuccess) return err;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  if (per_sm > 2) per_sm = 2;  // at most two 256-column tensor-memory allocations per SM
  long long grid = static_cast<long long>(per_sm) * device_sm_count();
  if (grid > tiles) grid = tiles;
  kernel<<<static_cast<int>(grid), kTcThreads, smem, stream>>>(p, tiles, timeouts);
  return cudaGetLastError();
}

#define QS_INSTANTIATE_PREFILL_TC(D, M, DI) \
  template cudaError_t launch_prefill_tc<D, M, DI>(const PrefillParams&, int, unsigned int*, cudaStream_t);

#define QS_INSTANTIATE_PREFILL(D)                                                   \
  template cudaError_t launch_prefill<D, false, false>(const PrefillParams&, int, cudaStream_t); \
  template cudaError_t launch_prefill<D, true, false>(const PrefillParams&, int, cudaStream_t);  \
  template cudaError_t launch_prefill<D, false, true>(const PrefillParams&, int, cudaStream_t);  \
  template cudaError_t launch_prefill<D, true, true>(const PrefillParams&, int, cudaStream_t);   \
  QS_INSTANTIATE_PREFILL_TC(D, 64, false) QS_INSTANTIATE_PREFILL_TC(D, 64, true)          \
  QS_INSTANTIATE_PREFILL_TC(D, 128, false) QS_INSTANTIATE_PREFILL_TC(D, 128, true)

}  // namespace qs
