// merge.cu -- standalone online-softmax fold and gradient fold (bandwidth
// kernels).
//
// [Ring-page] "Technical insight": block results are combined through a
// running max and running normaliser, earlier partial sums being rescaled when
// a larger max appears. For two partials over disjoint key sets with
// normalisers LSE_a, LSE_b (natural log) and normalised outputs O_a, O_b:
//   m = max(LSE_a, LSE_b),  LSE = m + log(exp(LSE_a - m) + exp(LSE_b - m)),
//   O = exp(LSE_a - LSE) O_a + exp(LSE_b - LSE) O_b.
// Each thread owns one 16-byte vector of a row; the row's weights are
// recomputed per thread from the two LSE words (both cached).
#include <math.h>

#include "internal.h"

namespace rattn {
namespace {

// When a row's vectors all live in one warp (D/4 divides 32) the row's LSE is
// written by its first thread after every thread of the row has read it;
// otherwise a second pass (merge_lse_kernel) writes the LSE.
__global__ void merge_kernel(float4* __restrict__ o_acc, float* __restrict__ lse_acc,
                             const float4* __restrict__ o_blk, const float* __restrict__ lse_blk, long long rows,
                             int vec_per_row, int write_lse) {
  const long long total = rows * vec_per_row;
  for (long long v = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; v < total;
       v += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = v / vec_per_row;
    const int e = static_cast<int>(v - row * vec_per_row);
    const float a = lse_acc[row];
    const float b = __ldg(lse_blk + row);
    const float m = fmaxf(a, b);
    float ca = 0.f, cb = 0.f, lse = -INFINITY;
    if (m != -INFINITY) {
      const float wa = expf(a - m);
      const float wb = expf(b - m);
      const float tot = wa + wb;
      lse = m + logf(tot);
      ca = wa / tot;
      cb = wb / tot;
    }
    const float4 x = o_acc[v];
    const float4 y = __ldg(o_blk + v);
    o_acc[v] = make_float4(ca * x.x + cb * y.x, ca * x.y + cb * y.y, ca * x.z + cb * y.z, ca * x.w + cb * y.w);
    if (write_lse) {
      __syncwarp(__activemask());
      if (e == 0) lse_acc[row] = lse;
    }
  }
}

__global__ void merge_lse_kernel(float* __restrict__ lse_acc, const float* __restrict__ lse_blk, long long rows) {
  for (long long r = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; r < rows;
       r += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float a = lse_acc[r];
    const float b = __ldg(lse_blk + r);
    const float m = fmaxf(a, b);
    lse_acc[r] = m == -INFINITY ? -INFINITY : m + logf(expf(a - m) + expf(b - m));
  }
}

unsigned grid_for(long long work, int threads) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (work + threads - 1) / threads;
  const long long cap = static_cast<long long>(sms) * 16;
  return static_cast<unsigned>(want < cap ? (want > 0 ? want : 1) : cap);
}

// acc += blk over n4 16-byte vectors (the running dK / dV sums of the ring
// backward across processes).
__global__ void grad_fold_kernel(float4* __restrict__ acc, const float4* __restrict__ blk, long long n4) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 a = acc[i];
    const float4 b = __ldg(blk + i);
    acc[i] = make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
  }
}

}  // namespace

rattn_status launch_grad_fold(float* acc, const float* blk, int64_t n, cudaStream_t stream) {
  const long long n4 = n / 4;
  grad_fold_kernel<<<grid_for(n4, 256), 256, 0, stream>>>(reinterpret_cast<float4*>(acc),
                                                          reinterpret_cast<const float4*>(blk), n4);
  return cudaGetLastError() == cudaSuccess ? RATTN_OK : RATTN_ERR_CUDA;
}

rattn_status launch_merge(float* o_acc, float* lse_acc, const float* o_blk, const float* lse_blk, int64_t rows, int D,
                          cudaStream_t stream) {
  const int vpr = D / 4;
  const int fused = (32 % vpr) == 0;
  merge_kernel<<<grid_for(rows * vpr, 256), 256, 0, stream>>>(reinterpret_cast<float4*>(o_acc), lse_acc,
                                                              reinterpret_cast<const float4*>(o_blk), lse_blk, rows,
                                                              vpr, fused);
  if (cudaGetLastError() != cudaSuccess) return RATTN_ERR_CUDA;
  if (fused) return RATTN_OK;
  merge_lse_kernel<<<grid_for(rows, 256), 256, 0, stream>>>(lse_acc, lse_blk, rows);
  return cudaGetLastError() == cudaSuccess ? RATTN_OK : RATTN_ERR_CUDA;
}

}  // namespace rattn
