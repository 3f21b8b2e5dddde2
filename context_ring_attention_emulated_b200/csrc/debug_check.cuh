// debug_check.cuh -- device-side bounds checks of the debug build.
//
// Built with -DRATTN_DEBUG (python -m context_ring_attention_emulated_b200.build
// --debug, which writes librattn_debug.so), every global-memory index that a
// kernel computes itself (position and segment-id reads, LSE / Delta reads,
// O, LSE, dK and dV writes) is checked against the extent of its array before
// the access. A failed check records SITE_BOUNDS + the check's number in the
// device error word (the first failure wins; rattn_get_device_error reports it
// as RATTN_ERR_BOUNDS) and the access is skipped, never trapped. In the normal
// build the checks compile to nothing. TMA copies need no such check: the
// tensor maps bound them in hardware.
#pragma once

#include "internal.h"

namespace rattn {

#ifdef RATTN_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif

// Whether index i lies in [0, n); in a debug build a miss is recorded as
// check `id` (always true otherwise).
__device__ __forceinline__ bool in_bounds(long long i, long long n, int* err, int id) {
  if constexpr (!kDebugChecks) {
    return true;
  } else {
    if (i >= 0 && i < n) return true;
    if (err) atomicCAS(err, 0, SITE_BOUNDS + id);
    return false;
  }
}

// Debug builds also check the ordering the kernels rely on: positions must be
// non-decreasing along every segment (rank slice). `ok` is the caller's
// comparison of a row's position with the previous row's; a violation is
// recorded as check `id`.
__device__ __forceinline__ void check_order(bool ok, int* err, int id) {
  if constexpr (kDebugChecks) {
    if (!ok && err) atomicCAS(err, 0, SITE_BOUNDS + id);
  }
}

}  // namespace rattn
