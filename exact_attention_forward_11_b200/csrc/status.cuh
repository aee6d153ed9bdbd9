// status.cuh - the library's device status word and the debug build's checks.
//
// A kernel whose bounded wait ran out ORs kStatusTimeout into g_status;
// attn_get_device_status reads and clears it. One word per device for the whole
// library: every stream, thread and entry point shares it.
//
// Built with -DATTN_DEBUG, the kernels also check their global-memory indices
// and TMA coordinates before each access (dbg_ok): a check that fails ORs
// kStatusBounds into g_status, records its site and index (the first failure
// since the last read wins) and returns false, and the caller skips the access.
// Nothing traps. Without ATTN_DEBUG dbg_ok is the constant true and the checks
// compile away.
#pragma once

#include <cstdint>

namespace attn {

constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusBounds = 2u;

#ifdef ATTN_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif

// Sites of the debug checks (reported by attn_debug_last_failure).
enum DebugSite : uint32_t {
  kSiteNone = 0,
  kSiteFwdOut = 1,         // O row and LSE store, two-Q-tile forward
  kSiteFwd1Out = 2,        // O row and LSE store, one-Q-tile forward
  kSiteFwd1ScaleLoad = 3,  // MXFP8 scale-byte load, one-Q-tile forward
  kSiteBwdDkDv = 4,        // dK / dV row store
  kSiteBwdStats = 5,       // LSE / D_i load of the dK dV kernel
  kSiteBwdDq = 6,          // dQ kernel row: LSE / D_i load and dQ store
  kSiteFp8Scale = 7,       // tile scale store, FP8 preparation
  kSiteMxBlock = 8,        // code / scale-byte store, MXFP8 quantisation
  kSiteW4Out = 9,          // output column store, W4A16 GEMM
  kSiteTmaCoord = 10,      // TMA coordinate (x not a multiple of 16 elements, a negative store
                           // coordinate, or a unit outside the launch)
  kSiteW4Split = 11,       // partial slot or ticket index, split-K W4A16 GEMM
};

__device__ uint32_t g_status;
__device__ uint32_t g_debug_site;       // first failing check's site since the last read
__device__ unsigned long long g_debug_index;   // and the index it rejected

__device__ __forceinline__ void record_timeout() { atomicOr(&g_status, kStatusTimeout); }

// true if the access may go ahead. Debug builds: `ok` is the check's verdict;
// a failure is recorded with `site` and `index`.
__device__ __forceinline__ bool dbg_ok(bool ok, uint32_t site, unsigned long long index) {
  if constexpr (!kDebugChecks) {
    return true;
  } else {
    if (!ok) {
      atomicOr(&g_status, kStatusBounds);
      if (atomicCAS(&g_debug_site, 0u, site) == 0u) atomicExch(&g_debug_index, index);
    }
    return ok;
  }
}

}  // namespace attn
