// status.cuh -- status codes shared by the kernels and the C ABI (from the public header).
#pragma once

#include "moe_b200.h"

namespace moe {

// Byte size of the workspace header: the device status word at byte 0, the
// permutation's completion counter at kWsCounterOffset, the GEMM's tile and exit
// counters at kWsTileCtrOffset (+4), the fused gate GEMV's completion counter at
// kWsGateCtrOffset. All are zero when idle and left at zero.
constexpr size_t kWsHeader = 256;
constexpr size_t kWsCounterOffset = 64;
constexpr size_t kWsTileCtrOffset = 128;
constexpr size_t kWsGateCtrOffset = 192;

// Record the first device-side error in the status word (later errors keep the first).
__device__ __forceinline__ void set_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

}  // namespace moe
