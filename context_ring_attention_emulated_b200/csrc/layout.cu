// layout.cu -- context-parallel layout permute / unpermute (bandwidth kernels).
//
// [Megatron-CP] "Symmetric chunk assignment": the padded sequence of Lp
// tokens is cut into 2*cp chunks of c = Lp/(2*cp); rank r holds chunk r
// followed by chunk 2*cp-1-r, ranks concatenated in rank order, and every slot
// keeps its global position id. CONTIGUOUS (the naive split) is the identity.
// STRIPED ([Ring-page], striped attention) gives token g to rank g mod cp.
// Padding goes at the tail of the global sequence and is zero-filled.
//
// Both kernels are gathers: each thread moves 16-byte vectors of one output
// row, so stores are fully coalesced and loads are coalesced within a row.
// Rows wider than 4 KB (256 vectors) are not supported.
#include "cp_map.cuh"
#include "internal.h"

namespace rattn {
namespace {

// Thread layout: vpr consecutive threads move one row (vpr = row bytes / 16),
// blockDim.x / vpr rows per block step; blockIdx.y walks (batch, head). All
// per-vector index math is 32-bit; only the final offsets are 64-bit.
__global__ void permute_kernel(const uint4* __restrict__ x, uint4* __restrict__ y, int32_t* __restrict__ pos,
                               int BH, int L, int Lp, int vpr, int c, int cp, int layout) {
  const int e = threadIdx.x % vpr;
  const int rsub = threadIdx.x / vpr;
  const int rpb = blockDim.x / vpr;
  if (rsub >= rpb) return;
  for (int bh = blockIdx.y; bh < BH; bh += gridDim.y) {
    const uint4* xb = x + static_cast<long long>(bh) * L * vpr;
    uint4* yb = y + static_cast<long long>(bh) * Lp * vpr;
    for (int i = blockIdx.x * rpb + rsub; i < Lp; i += gridDim.x * rpb) {
      const int g = slot_to_global(i, c, cp, layout);
      uint4 val = make_uint4(0u, 0u, 0u, 0u);
      if (g < L) val = __ldg(xb + static_cast<long long>(g) * vpr + e);
      yb[static_cast<long long>(i) * vpr + e] = val;
      if (pos && bh == 0 && e == 0) pos[i] = g;
    }
  }
}

__global__ void unpermute_kernel(const uint4* __restrict__ y, uint4* __restrict__ x, int BH, int L, int Lp,
                                 int vpr, int c, int cp, int layout) {
  const int e = threadIdx.x % vpr;
  const int rsub = threadIdx.x / vpr;
  const int rpb = blockDim.x / vpr;
  if (rsub >= rpb) return;
  for (int bh = blockIdx.y; bh < BH; bh += gridDim.y) {
    const uint4* yb = y + static_cast<long long>(bh) * Lp * vpr;
    uint4* xb = x + static_cast<long long>(bh) * L * vpr;
    for (int g = blockIdx.x * rpb + rsub; g < L; g += gridDim.x * rpb) {
      const int i = global_to_slot(g, c, cp, layout);
      xb[static_cast<long long>(g) * vpr + e] = __ldg(yb + static_cast<long long>(i) * vpr + e);
    }
  }
}

// Varlen gather: y[bh][i] = src[i] in [0, T_in) ? x[bh][src[i]] : 0.
__global__ void gather_kernel(const uint4* __restrict__ x, uint4* __restrict__ y, const int32_t* __restrict__ src,
                              int BH, int T_in, int T_out, int vpr) {
  const int e = threadIdx.x % vpr;
  const int rsub = threadIdx.x / vpr;
  const int rpb = blockDim.x / vpr;
  if (rsub >= rpb) return;
  for (int bh = blockIdx.y; bh < BH; bh += gridDim.y) {
    const uint4* xb = x + static_cast<long long>(bh) * T_in * vpr;
    uint4* yb = y + static_cast<long long>(bh) * T_out * vpr;
    for (int i = blockIdx.x * rpb + rsub; i < T_out; i += gridDim.x * rpb) {
      const int g = __ldg(src + i);
      uint4 val = make_uint4(0u, 0u, 0u, 0u);
      if (g >= 0 && g < T_in) val = __ldg(xb + static_cast<long long>(g) * vpr + e);
      yb[static_cast<long long>(i) * vpr + e] = val;
    }
  }
}

// Varlen scatter: x[bh][src[i]] = y[bh][i] for src[i] in [0, T_x).
__global__ void scatter_kernel(const uint4* __restrict__ y, uint4* __restrict__ x, const int32_t* __restrict__ src,
                               int BH, int T_y, int T_x, int vpr) {
  const int e = threadIdx.x % vpr;
  const int rsub = threadIdx.x / vpr;
  const int rpb = blockDim.x / vpr;
  if (rsub >= rpb) return;
  for (int bh = blockIdx.y; bh < BH; bh += gridDim.y) {
    const uint4* yb = y + static_cast<long long>(bh) * T_y * vpr;
    uint4* xb = x + static_cast<long long>(bh) * T_x * vpr;
    for (int i = blockIdx.x * rpb + rsub; i < T_y; i += gridDim.x * rpb) {
      const int g = __ldg(src + i);
      if (g >= 0 && g < T_x) xb[static_cast<long long>(g) * vpr + e] = __ldg(yb + static_cast<long long>(i) * vpr + e);
    }
  }
}

// Grid for rows x BH work items: about 16 resident 256-thread blocks per SM.
dim3 grid_2d(long long rows, int BH, int rpb) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int gy = BH < 65535 ? BH : 65535;
  const long long want_total = static_cast<long long>(sms) * 16;
  long long gx = (want_total + gy - 1) / gy;
  const long long row_blocks = (rows + rpb - 1) / rpb;
  if (gx > row_blocks) gx = row_blocks;
  if (gx < 1) gx = 1;
  return dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy), 1);
}


}  // namespace

rattn_status launch_gather(const void* x, void* y, const int32_t* src, int BH, int64_t T_in, int64_t T_out,
                           int row_bytes, cudaStream_t stream) {
  const int vpr = row_bytes / 16;
  if (vpr > 256) return RATTN_ERR_UNSUPPORTED;
  gather_kernel<<<grid_2d(T_out, BH, 256 / vpr), 256, 0, stream>>>(
      static_cast<const uint4*>(x), static_cast<uint4*>(y), src, BH, static_cast<int>(T_in), static_cast<int>(T_out),
      vpr);
  return cudaGetLastError() == cudaSuccess ? RATTN_OK : RATTN_ERR_CUDA;
}

rattn_status launch_scatter(const void* y, void* x, const int32_t* src, int BH, int64_t T_y, int64_t T_x,
                            int row_bytes, cudaStream_t stream) {
  const int vpr = row_bytes / 16;
  if (vpr > 256) return RATTN_ERR_UNSUPPORTED;
  scatter_kernel<<<grid_2d(T_y, BH, 256 / vpr), 256, 0, stream>>>(
      static_cast<const uint4*>(y), static_cast<uint4*>(x), src, BH, static_cast<int>(T_y), static_cast<int>(T_x),
      vpr);
  return cudaGetLastError() == cudaSuccess ? RATTN_OK : RATTN_ERR_CUDA;
}

rattn_status launch_permute(const void* x, void* y, int32_t* pos, int BH, int64_t L, int64_t Lp, int row_bytes,
                            int cp, int layout, cudaStream_t stream) {
  const int vpr = row_bytes / 16;
  const int c = cp_map_c(Lp, cp, layout);
  if (vpr > 256) return RATTN_ERR_UNSUPPORTED;
  permute_kernel<<<grid_2d(Lp, BH, 256 / vpr), 256, 0, stream>>>(static_cast<const uint4*>(x), static_cast<uint4*>(y),
                                                                 pos, BH, static_cast<int>(L), static_cast<int>(Lp),
                                                                 vpr, c, cp, layout);
  return cudaGetLastError() == cudaSuccess ? RATTN_OK : RATTN_ERR_CUDA;
}

rattn_status launch_unpermute(const void* y, void* x, int BH, int64_t L, int64_t Lp, int row_bytes, int cp,
                              int layout, cudaStream_t stream) {
  const int vpr = row_bytes / 16;
  const int c = cp_map_c(Lp, cp, layout);
  if (vpr > 256) return RATTN_ERR_UNSUPPORTED;
  unpermute_kernel<<<grid_2d(L, BH, 256 / vpr), 256, 0, stream>>>(static_cast<const uint4*>(y),
                                                                  static_cast<uint4*>(x), BH, static_cast<int>(L),
                                                                  static_cast<int>(Lp), vpr, c, cp, layout);
  return cudaGetLastError() == cudaSuccess ? RATTN_OK : RATTN_ERR_CUDA;
}

}  // namespace rattn
