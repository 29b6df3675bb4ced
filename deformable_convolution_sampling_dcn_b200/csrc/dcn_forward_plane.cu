// Shared-memory forward path (placeholder until the staged kernel lands).
#include "dcn_launch.h"

namespace dcnb {
cudaError_t launch_core_forward_plane(const CoreArgs &, cudaStream_t, bool *handled) {
    *handled = false;
    return cudaSuccess;
}
}  // namespace dcnb
