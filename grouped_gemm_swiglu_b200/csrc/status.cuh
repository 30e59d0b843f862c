// status.cuh -- status codes shared by the kernels and the C ABI (from the public header).
#pragma once

#include "moe_b200.h"

namespace moe {

// Byte size of the workspace header that holds the device status word.
constexpr size_t kWsHeader = 256;

// Record the first device-side error in the status word (later errors keep the first).
__device__ __forceinline__ void set_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

}  // namespace moe
