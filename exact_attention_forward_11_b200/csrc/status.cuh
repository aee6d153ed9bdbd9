// status.cuh - the library's device status word.
//
// A kernel whose bounded wait ran out ORs kStatusTimeout into g_status;
// attn_get_device_status reads and clears it. One word per device for the whole
// library: every stream, thread and entry point shares it.
#pragma once

#include <cstdint>

namespace attn {

constexpr uint32_t kStatusTimeout = 1u;

__device__ uint32_t g_status;

__device__ __forceinline__ void record_timeout() { atomicOr(&g_status, kStatusTimeout); }

}  // namespace attn
