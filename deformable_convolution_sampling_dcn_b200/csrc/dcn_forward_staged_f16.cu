// Staged forward kernels for __half storage (see dcn_forward_staged.cuh).
#include "dcn_forward_staged.cuh"

namespace dcnb {
DCNB_STAGED_INSTANCE(__half)
}  // namespace dcnb
