// cp_map.cuh -- slot <-> global-position maps of the context-parallel layouts.
//
// [Megatron-CP] "Symmetric chunk assignment" (HEAD_TAIL): the padded sequence
// of Lp tokens is cut into 2*cp chunks of c = Lp/(2*cp); rank r holds chunk r
// followed by chunk 2*cp-1-r, ranks concatenated in rank order. CONTIGUOUS
// (the naive split) is the identity. STRIPED ([Ring-page], striped attention)
// gives token g to rank g mod cp; c is then the per-rank length Lp / cp.
#pragma once

#include "rattn.h"

namespace rattn {

// Global position held by slot i of the permuted sequence.
__host__ __device__ __forceinline__ int slot_to_global(int i, int c, int cp, int layout) {
  if (layout == RATTN_LAYOUT_CONTIGUOUS) return i;
  if (layout == RATTN_LAYOUT_STRIPED) {
    const int r = i / c;
    return (i - r * c) * cp + r;
  }
  const int r = i / (2 * c);
  const int j = i - r * 2 * c;
  return j < c ? r * c + j : (2 * cp - 1 - r) * c + (j - c);
}

// Slot of the permuted sequence that holds global position g.
__host__ __device__ __forceinline__ int global_to_slot(int g, int c, int cp, int layout) {
  if (layout == RATTN_LAYOUT_CONTIGUOUS) return g;
  if (layout == RATTN_LAYOUT_STRIPED) {
    const int j = g / cp;
    return (g - j * cp) * c + j;
  }
  const int k = g / c;
  const int j = g - k * c;
  return k < cp ? k * 2 * c + j : (2 * cp - 1 - k) * 2 * c + c + j;
}

// c as the maps above take it: chunk length (HEAD_TAIL) or per-rank length.
inline int cp_map_c(long long Lp, int cp, int layout) {
  return static_cast<int>(Lp / (layout == RATTN_LAYOUT_HEAD_TAIL ? 2 * cp : cp));
}

}  // namespace rattn
