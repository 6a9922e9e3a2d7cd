// common.cuh -- shared device definitions of libmoe (single translation unit).
#pragma once

#include <cstdint>

#include "../../include/moe.h"
#include "ptx.cuh"

namespace moe {

// Per-device status word (MOE_STATUS_* bits), read and cleared by
// moe_get_device_status.  Kernels only ever OR bits into it.
__device__ unsigned int g_status;

__device__ __forceinline__ void flag_status(unsigned int bits) { atomicOr(&g_status, bits); }

}  // namespace moe
