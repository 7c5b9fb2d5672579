// Chunkwise prefill kernel instances (Dk = 64, 128; scalar and diagonal decay).
#include "qstate_launch_prefill_impl.cuh"

namespace qs {
QS_INSTANTIATE_PREFILL(64)
QS_INSTANTIATE_PREFILL(128)
}  // namespace qs
