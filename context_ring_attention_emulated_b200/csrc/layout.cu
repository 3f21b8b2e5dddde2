// layout.cu -- context-parallel layout permute / unpermute (bandwidth kernels).
//
// [Megatron-CP] "Symmetric chunk assignment": the padded sequence of Lp
// tokens is cut into 2*cp chunks of c = Lp/(2*cp); rank r holds chunk r
// followed by chunk 2*cp-1-r, ranks concatenated in rank order, and every slot
// keeps its global position id. CONTIGUOUS (the naive split) is the identity.
// Padding goes at the tail of the global sequence and is zero-filled.
//
// Both kernels are gathers: each thread moves 16-byte vectors of one output
// row, so stores are fully coalesced and loads are coalesced within a row.
#include "internal.h"

namespace rattn {
namespace {

// Global position held by slot i of the permuted sequence.
__device__ __forceinline__ int slot_to_global(int i, int c, int cp, int layout) {
  if (layout == RATTN_LAYOUT_CONTIGUOUS) return i;
  const int r = i / (2 * c);
  const int j = i - r * 2 * c;
  return j < c ? r * c + j : (2 * cp - 1 - r) * c + (j - c);
}

// Slot of the permuted sequence that holds global position g.
__device__ __forceinline__ int global_to_slot(int g, int c, int cp, int layout) {
  if (layout == RATTN_LAYOUT_CONTIGUOUS) return g;
  const int k = g / c;
  const int j = g - k * c;
  return k < cp ? k * 2 * c + j : (2 * cp - 1 - k) * 2 * c + c + j;
}

__global__ void permute_kernel(const uint4* __restrict__ x, uint4* __restrict__ y, int32_t* __restrict__ pos,
                               int BH, int L, int Lp, int vec_per_row, int c, int cp, int layout) {
  const long long total = static_cast<long long>(BH) * Lp * vec_per_row;
  for (long long v = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; v < total;
       v += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = v / vec_per_row;
    const int e = static_cast<int>(v - row * vec_per_row);
    const int bh = static_cast<int>(row / Lp);
    const int i = static_cast<int>(row - static_cast<long long>(bh) * Lp);
    const int g = slot_to_global(i, c, cp, layout);
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (g < L) val = __ldg(x + (static_cast<long long>(bh) * L + g) * vec_per_row + e);
    y[v] = val;
    if (pos && bh == 0 && e == 0) pos[i] = g;
  }
}

__global__ void unpermute_kernel(const uint4* __restrict__ y, uint4* __restrict__ x, int BH, int L, int Lp,
                                 int vec_per_row, int c, int cp, int layout) {
  const long long total = static_cast<long long>(BH) * L * vec_per_row;
  for (long long v = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; v < total;
       v += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = v / vec_per_row;
    const int e = static_cast<int>(v - row * vec_per_row);
    const int bh = static_cast<int>(row / L);
    const int g = static_cast<int>(row - static_cast<long long>(bh) * L);
    const int i = global_to_slot(g, c, cp, layout);
    x[v] = __ldg(y + (static_cast<long long>(bh) * Lp + i) * vec_per_row + e);
  }
}

unsigned grid_for(long long work, int threads) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (work + threads - 1) / threads;
  const long long cap = static_cast<long long>(sms) * 16;  // 16 resident 256-thread CTAs per SM
  return static_cast<unsigned>(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

rattn_status launch_permute(const void* x, void* y, int32_t* pos, int BH, int64_t L, int64_t Lp, int row_bytes,
                            int cp, int layout, cudaStream_t stream) {
  const int vpr = row_bytes / 16;
  const int nchunks = layout == RATTN_LAYOUT_HEAD_TAIL ? 2 * cp : cp;
  const int c = static_cast<int>(Lp / nchunks);
  const long long total = static_cast<long long>(BH) * Lp * vpr;
  permute_kernel<<<grid_for(total, 256), 256, 0, stream>>>(static_cast<const uint4*>(x), static_cast<uint4*>(y), pos,
                                                           BH, static_cast<int>(L), static_cast<int>(Lp), vpr, c, cp,
                                                           layout);
  return cudaGetLastError() == cudaSuccess ? RATTN_OK : RATTN_ERR_CUDA;
}

rattn_status launch_unpermute(const void* y, void* x, int BH, int64_t L, int64_t Lp, int row_bytes, int cp,
                              int layout, cudaStream_t stream) {
  const int vpr = row_bytes / 16;
  const int nchunks = layout == RATTN_LAYOUT_HEAD_TAIL ? 2 * cp : cp;
  const int c = static_cast<int>(Lp / nchunks);
  const long long total = static_cast<long long>(BH) * L * vpr;
  unpermute_kernel<<<grid_for(total, 256), 256, 0, stream>>>(static_cast<const uint4*>(y), static_cast<uint4*>(x),
                                                             BH, static_cast<int>(L), static_cast<int>(Lp), vpr, c,
                                                             cp, layout);
  return cudaGetLastError() == cudaSuccess ? RATTN_OK : RATTN_ERR_CUDA;
}

}  // namespace rattn
