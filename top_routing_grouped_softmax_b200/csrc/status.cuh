// status.cuh -- the per-device status word that kernels write when they
// detect an error (index data out of range, a pipeline wait past its limit,
// a value outside the range of its storage type),
// and the per-device wait limit.  The library is built as one translation
// unit, so these definitions exist once per device.
#pragma once

#include <cstdint>

namespace moe {

// Values match moe_status_t in include/moe.h.
constexpr int kStatusOk = 0;
constexpr int kStatusDeviceTimeout = 5;
constexpr int kStatusDeviceBounds = 6;
constexpr int kStatusDeviceRange = 9;

__device__ int g_status = 0;
__device__ unsigned long long g_wait_limit_ns = 1000000000ull;

// Keep the first error recorded since the host last cleared the word.
__device__ __forceinline__ void record_status(int code)
{
    atomicCAS(&g_status, kStatusOk, code);
}

}  // namespace moe
