// fwd_positions.cuh -- position and segid lookups shared by the attention
// forward kernels. P is the kernel's parameter block: q_pos, kv_pos (global
// position per slot, or NULL for the row index), seg (segid per slot for
// packed sequences), nseg, Lq_seg, Lk_seg and the device error word err.
// Every index is checked by the debug build before the load (debug_check.cuh).
#pragma once

#include "debug_check.cuh"

namespace rattn {

// Global position of query row `row` of segment (rank) `seg`.
template <class P>
__device__ __forceinline__ long long qpos(const P& p, int seg, int row) {
  const long long i = static_cast<long long>(seg) * p.Lq_seg + row;
  if (!in_bounds(i, static_cast<long long>(p.nseg) * p.Lq_seg, p.err, 1)) return 0;
  return p.q_pos ? static_cast<long long>(__ldg(p.q_pos + i)) : row;
}

// Global position of key row `row` of segment (rank) `seg`.
template <class P>
__device__ __forceinline__ long long kpos(const P& p, int seg, int row) {
  const long long i = static_cast<long long>(seg) * p.Lk_seg + row;
  if (!in_bounds(i, static_cast<long long>(p.nseg) * p.Lk_seg, p.err, 2)) return 0;
  return p.kv_pos ? static_cast<long long>(__ldg(p.kv_pos + i)) : row;
}

// segid of a slot (packed sequences; only called when p.seg is set). Query and
// key slots share one array (rank-major, Lq_seg == Lk_seg in ring calls).
template <class P>
__device__ __forceinline__ int segat(const P& p, int rank, int row) {
  const long long i = static_cast<long long>(rank) * p.Lk_seg + row;
  if (!in_bounds(i, static_cast<long long>(p.nseg) * p.Lk_seg, p.err, 3)) return 1;
  return __ldg(p.seg + i);
}

}  // namespace rattn
