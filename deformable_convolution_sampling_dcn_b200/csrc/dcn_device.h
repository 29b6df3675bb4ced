// Per-device facts and the driver's tensor-map encoder, shared by the
// launchers that build TMA descriptors.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

namespace dcnb {

struct DeviceInfo {
    int sms = 0, smem_optin = 0, smem_per_sm = 0;
    unsigned int *err = nullptr;  // device error word (bit 0: a bounded wait ran out)
};

// Facts of the current device, looked up once per device (the error word's
// address is per device context).  nullptr if they cannot be obtained.
const DeviceInfo *device_info();

// cuTensorMapEncodeTiled from the driver, or nullptr.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn();

}  // namespace dcnb
