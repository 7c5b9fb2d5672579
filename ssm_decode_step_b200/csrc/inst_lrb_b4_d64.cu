// Low-Rank Bypass kernel instances for 4-bit codes and Dk = 64.
#include "qstate_launch_impl.cuh"

namespace qs {
QS_INSTANTIATE_LRB(4, 64)
}  // namespace qs
