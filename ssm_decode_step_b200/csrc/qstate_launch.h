// Host-side launchers of the decode-step kernels, one per compile-time
// configuration.  Defined in qstate_launch_impl.cuh and instantiated in the
// inst_b*_d*.cu files (one translation unit per bit width and key size, so
// they compile in parallel).
#pragma once

#include <cuda_runtime.h>

#include "qstate_kernels.cuh"
#include "qstate_step.cuh"
#include "qstate_stream.cuh"
#include "qstate_lrb.cuh"
#include "qstate_lrb_stream.cuh"

namespace qs {

template <int BITS, int DK, int POLICY, bool BDR, bool DELTA, bool DIAG>
cudaError_t launch_step(const StepParams& p, cudaStream_t stream);

template <int BITS, int DK>
cudaError_t launch_readout(const StepParams& p, cudaStream_t stream);

// Low-Rank Bypass step; p carries pointers, group, rank, rpad and slot.
template <int BITS, int DK, int POLICY, bool BDR, bool DELTA, bool DIAG, bool MERGE>
cudaError_t launch_lrb(const LrbParams& p, int tiles, int dv, cudaStream_t stream);

template <int BITS, int DK>
cudaError_t launch_init(const float* S0, uint8_t* codes, float* scales, float* shadow,
                        long long rows, int group, cudaStream_t stream);

// Streaming multiprocessors of the current device (queried once per device).
int device_sm_count();

}  // namespace qs
