// Staged forward kernels for float storage (see dcn_forward_staged.cuh).
#include "dcn_forward_staged.cuh"

namespace dcnb {
DCNB_STAGED_INSTANCE(float)
}  // namespace dcnb
