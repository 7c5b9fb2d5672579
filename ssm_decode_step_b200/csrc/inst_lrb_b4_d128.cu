// Low-Rank Bypass kernel instances for 4-bit codes and Dk = 128.
#include "qstate_launch_impl.cuh"

namespace qs {
QS_INSTANTIATE_LRB(4, 128)
}  // namespace qs
