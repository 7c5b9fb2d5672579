// Kernel instances for 4-bit codes and Dk = 64.
#include "qstate_launch_impl.cuh"

namespace qs {
QS_INSTANTIATE_ALL(4, 64)
}  // namespace qs
