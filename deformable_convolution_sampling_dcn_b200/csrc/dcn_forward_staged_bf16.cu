// Staged forward kernels for __nv_bfloat16 storage (see dcn_forward_staged.cuh).
#include "dcn_forward_staged.cuh"

namespace dcnb {
DCNB_STAGED_INSTANCE(__nv_bfloat16)
}  // namespace dcnb
