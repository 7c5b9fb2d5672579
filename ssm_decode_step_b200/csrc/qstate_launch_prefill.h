// Host-side launchers of the chunkwise prefill kernels.  Defined in
// qstate_launch_prefill_impl.cuh and instantiated in inst_prefill.cu, apart
// from the decode-step launchers so that the two evolve independently.
#pragma once

#include <cuda_runtime.h>

#include "qstate_prefill.cuh"
#include "qstate_prefill_tc.cuh"

namespace qs {

// Chunkwise prefill (linear write or delta rule) of `tiles` tiles.
template <int DK, bool DIAG, bool DELTA>
cudaError_t launch_prefill(const PrefillParams& p, int tiles, cudaStream_t stream);

// Chunkwise prefill on the tensor cores (TF32 operands, FP32 accumulators);
// MDV = 64 or 128 accumulator rows (dv <= MDV); timeouts counts CTAs whose
// bounded wait for the tensor cores gave up.
template <int DK, int MDV, bool DIAG>
cudaError_t launch_prefill_tc(const PrefillParams& p, int tiles, unsigned int* timeouts,
                              cudaStream_t stream);

}  // namespace qs
