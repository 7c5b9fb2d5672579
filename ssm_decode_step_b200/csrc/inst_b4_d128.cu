// Kernel instances for 4-bit codes and Dk = 128.
#include "qstate_launch_impl.cuh"

namespace qs {
QS_INSTANTIATE_ALL(4, 128)
}  // namespace qs
