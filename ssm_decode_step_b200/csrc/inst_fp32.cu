// Kernel instances of the unquantized FP32 decode step.
#include <mutex>

#include "qstate_fp32.cuh"
#include "qstate_launch_impl.cuh"

namespace qs {

template <int DK, bool DELTA, bool DIAG>
cudaError_t launch_fp32_step(const StepParams& p0, cudaStream_t stream) {
  constexpr int S = 3;
  auto kernel = fp32_step_kernel<DK, DELTA, DIAG, S>;
  static std::once_flag flag;
  cudaError_t err = allow_smem(kernel, flag);
  if (err != cudaSuccess) return err;
  StepParams p = p0;
  // rows per unit: the largest of 32, 16 that divides dv (a stage of 16-18 KB)
  p.rb = p.dv % 32 == 0 ? 32 : 16;
  p.units_per_tile = p.dv / p.rb;
  const Fp32Layout L(DK, p.rb, DIAG);
  return launch_persistent(kernel, static_cast<size_t>(S) * L.bytes, p, stream);
}

template cudaError_t launch_fp32_step<64, false, false>(const StepParams&, cudaStream_t);
template cudaError_t launch_fp32_step<64, false, true>(const StepParams&, cudaStream_t);
template cudaError_t launch_fp32_step<64, true, false>(const StepParams&, cudaStream_t);
template cudaError_t launch_fp32_step<64, true, true>(const StepParams&, cudaStream_t);
template cudaError_t launch_fp32_step<128, false, false>(const StepParams&, cudaStream_t);
template cudaError_t launch_fp32_step<128, false, true>(const StepParams&, cudaStream_t);
template cudaError_t launch_fp32_step<128, true, false>(const StepParams&, cudaStream_t);
template cudaError_t launch_fp32_step<128, true, true>(const StepParams&, cudaStream_t);

}  // namespace qs
