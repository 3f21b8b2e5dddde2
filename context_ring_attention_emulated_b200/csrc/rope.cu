// rope.cu -- layout permute with rotary position embedding fused in, and the
// matching gradient unpermute (bandwidth kernels).
//
// [Megatron-CP] "Symmetric chunk assignment": RoPE must use every token's
// global position (a rank holding chunks r and 2*cp-1-r rotates with those
// chunks' positions, never with local indices). The rotation is RoFormer's
// (Su et al., 2021): pair i of a head vector turns by p * base^(-2i/D) at
// position p. HALF pairs (x[i], x[i + D/2]); INTERLEAVED pairs (x[2i], x[2i+1]).
//
// permute_rope:         y[slot(g)] = R(+theta_g) x[g]   (zero pad rows)
// unpermute_rope_grad:  dx[g]      = R(-theta_g) dy[slot(g)]
// (R is orthogonal, so the gradient through the rotation is the inverse
// rotation; fused into the unpermute of dQ / dK.)
//
// Thread layout: each thread owns whole rotation pairs of one row (one 16-B
// vector for INTERLEAVED; a vector and its partner D/2 elements later for
// HALF), computes their cos/sin once (angle in fp64, reduced modulo 2 pi,
// then fp32 sin/cos) and
// then walks (batch, head) with a stride of gridDim.y, so the trigonometry is
// amortised over the heads while every access stays a 16-byte vector.
#include <cuda_bf16.h>
#include <math.h>

#include "cp_map.cuh"
#include "internal.h"

namespace rattn {
namespace {

constexpr double k2Pi = 6.283185307179586;
constexpr double kInv2Pi = 0.15915494309189535;

template <typename T>
struct Vec;
template <>
struct Vec<float> {
  static constexpr int W = 4;  // elements per 16-byte vector
  __device__ static void load(const uint4& u, float (&f)[W]) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
  }
  __device__ static uint4 store(const float (&f)[W]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
  }
};
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int W = 8;
  __device__ static void load(const uint4& u, float (&f)[W]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[k]));
      f[2 * k] = t.x;
      f[2 * k + 1] = t.y;
    }
  }
  __device__ static uint4 store(const float (&f)[W]) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __nv_bfloat162 t = __floats2bfloat162_rn(f[2 * k], f[2 * k + 1]);
      w[k] = *reinterpret_cast<const uint32_t*>(&t);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};

struct RopeArgs {
  const uint4* src;
  uint4* dst;
  int32_t* pos;  // permute only; may be NULL
  int BH, L, Lp, D, c, cp, layout;
  int vpr;       // 16-byte vectors per row
  int tpr;       // threads per row
  float sign;    // +1 rotate, -1 inverse rotation
  double base;
};

// (x0[t], x1[t]) -> rotated pair t, for the W pairs of a HALF thread.
template <typename T, int NP>
__device__ __forceinline__ void rotate_half(const uint4& u0, const uint4& u1, const float (&cs)[NP],
                                            const float (&sn)[NP], uint4* out0, uint4* out1) {
  using V = Vec<T>;
  float x0[V::W], x1[V::W];
  V::load(u0, x0);
  V::load(u1, x1);
#pragma unroll
  for (int t = 0; t < V::W; ++t) {
    const float p = x0[t], q = x1[t];
    x0[t] = p * cs[t] - q * sn[t];
    x1[t] = p * sn[t] + q * cs[t];
  }
  *out0 = V::store(x0);
  *out1 = V::store(x1);
}

// (x[2t], x[2t+1]) -> rotated pair t, for the W/2 pairs of an INTERLEAVED thread.
template <typename T, int NP>
__device__ __forceinline__ void rotate_interleaved(const uint4& u, const float (&cs)[NP], const float (&sn)[NP],
                                                   uint4* out) {
  using V = Vec<T>;
  float x[V::W];
  V::load(u, x);
#pragma unroll
  for (int t = 0; t < V::W / 2; ++t) {
    const float p = x[2 * t], q = x[2 * t + 1];
    x[2 * t] = p * cs[t] - q * sn[t];
    x[2 * t + 1] = p * sn[t] + q * cs[t];
  }
  *out = V::store(x);
}

// PERMUTE: output rows are slots i (source row = its global position g);
// otherwise output rows are global positions g (source row = slot(g)).
template <typename T, int STYLE, bool PERMUTE>
__global__ void __launch_bounds__(256) rope_kernel(RopeArgs a) {
  using V = Vec<T>;
  constexpr int W = V::W;
  constexpr int NP = STYLE == RATTN_ROPE_HALF ? W : W / 2;  // pairs per thread
  extern __shared__ double s_invf[];                         // [D/2]
  const int half = a.D / 2;
  for (int k = threadIdx.x; k < half; k += blockDim.x)
    s_invf[k] = pow(a.base, -2.0 * static_cast<double>(k) / static_cast<double>(a.D));
  __syncthreads();

  const int e = threadIdx.x % a.tpr;
  const int rsub = threadIdx.x / a.tpr;
  const int rpb = blockDim.x / a.tpr;
  if (rsub >= rpb) return;
  const int n_out = PERMUTE ? a.Lp : a.L;
  const int n_src = PERMUTE ? a.L : a.Lp;
  // Vector indices of this thread's elements and the frequency index of its first pair.
  const int v0 = e;
  const int v1 = STYLE == RATTN_ROPE_HALF ? e + a.vpr / 2 : -1;
  const int k0 = STYLE == RATTN_ROPE_HALF ? e * W : e * (W / 2);

  for (int o = blockIdx.x * rpb + rsub; o < n_out; o += gridDim.x * rpb) {
    const int g = PERMUTE ? slot_to_global(o, a.c, a.cp, a.layout) : o;
    const int sr = PERMUTE ? g : global_to_slot(g, a.c, a.cp, a.layout);
    if (PERMUTE && a.pos && blockIdx.y == 0 && e == 0) a.pos[o] = g;
    const bool live = sr < n_src && g < a.L;
    float cs[NP], sn[NP];
    if (live) {
#pragma unroll
      for (int t = 0; t < NP; ++t) {
        // angle in fp64 (exact position times the frequency), reduced to
        // [-pi, pi] by subtracting the nearest multiple of 2 pi, then sin/cos
        // of the small fp32 remainder
        const double ang = static_cast<double>(g) * s_invf[k0 + t];
        const double red = fma(-rint(ang * kInv2Pi), k2Pi, ang);
        float sf, cf;
        sincosf(static_cast<float>(red), &sf, &cf);
        cs[t] = cf;
        sn[t] = a.sign * sf;
      }
    }
    // NR (batch, head) rows per step, all loads issued before any is used,
    // so every thread keeps four 16-byte loads in flight (HALF: two rows of
    // two vectors; INTERLEAVED: four rows of one vector).
    constexpr int NR = STYLE == RATTN_ROPE_HALF ? 2 : 4;
    for (int bh0 = blockIdx.y; bh0 < a.BH; bh0 += NR * gridDim.y) {
      const uint4* sp[NR];
      uint4* dp[NR];
      bool have[NR];
#pragma unroll
      for (int k = 0; k < NR; ++k) {
        const int bh = bh0 + k * gridDim.y;
        have[k] = bh < a.BH;
        const int b = have[k] ? bh : bh0;
        sp[k] = a.src + (static_cast<long long>(b) * n_src + sr) * a.vpr;
        dp[k] = a.dst + (static_cast<long long>(b) * n_out + o) * a.vpr;
      }
      if (!live) {
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int k = 0; k < NR; ++k) {
          if (!have[k]) continue;
          dp[k][v0] = z;
          if (STYLE == RATTN_ROPE_HALF) dp[k][v1] = z;
        }
        continue;
      }
      if (STYLE == RATTN_ROPE_HALF) {
        uint4 u0[NR], u1[NR];
#pragma unroll
        for (int k = 0; k < NR; ++k) {
          if (!have[k]) continue;
          u0[k] = __ldg(sp[k] + v0);
          u1[k] = __ldg(sp[k] + v1);
        }
#pragma unroll
        for (int k = 0; k < NR; ++k)
          if (have[k]) rotate_half<T, NP>(u0[k], u1[k], cs, sn, dp[k] + v0, dp[k] + v1);
      } else {
        uint4 u[NR];
#pragma unroll
        for (int k = 0; k < NR; ++k)
          if (have[k]) u[k] = __ldg(sp[k] + v0);
#pragma unroll
        for (int k = 0; k < NR; ++k)
          if (have[k]) rotate_interleaved<T, NP>(u[k], cs, sn, dp[k] + v0);
      }
    }
  }
}

// Rows along x (grid-stride), (batch, head) along y only as far as needed to
// fill the GPU (about 8 resident 256-thread blocks per SM), so each row's
// sin/cos are formed by as few blocks as possible.
dim3 rope_grid(long long rows, int BH, int rpb) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = static_cast<long long>(sms) * 8;
  long long gx = (rows + rpb - 1) / rpb;
  if (gx < 1) gx = 1;
  long long gy = 1;
  if (gx >= want) {
    gx = want;
  } else {
    gy = (want + gx - 1) / gx;
    if (gy > BH) gy = BH;
    if (gy > 65535) gy = 65535;
  }
  return dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy), 1);
}

template <typename T, int STYLE, bool PERMUTE>
rattn_status launch_one(RopeArgs a, cudaStream_t stream) {
  constexpr int W = Vec<T>::W;
  a.tpr = STYLE == RATTN_ROPE_HALF ? a.D / (2 * W) : a.D / W;
  const int rpb = 256 / a.tpr;
  const long long rows = PERMUTE ? a.Lp : a.L;
  const size_t smem = static_cast<size_t>(a.D / 2) * sizeof(double);
  rope_kernel<T, STYLE, PERMUTE><<<rope_grid(rows, a.BH, rpb), 256, smem, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? RATTN_OK : RATTN_ERR_CUDA;
}

template <bool PERMUTE>
rattn_status dispatch(RopeArgs a, rattn_dtype dtype, int style, cudaStream_t stream) {
  if (dtype == RATTN_BF16) {
    return style == RATTN_ROPE_HALF ? launch_one<__nv_bfloat16, RATTN_ROPE_HALF, PERMUTE>(a, stream)
                                    : launch_one<__nv_bfloat16, RATTN_ROPE_INTERLEAVED, PERMUTE>(a, stream);
  }
  return style == RATTN_ROPE_HALF ? launch_one<float, RATTN_ROPE_HALF, PERMUTE>(a, stream)
                                  : launch_one<float, RATTN_ROPE_INTERLEAVED, PERMUTE>(a, stream);
}

}  // namespace

rattn_status launch_permute_rope(const void* x, void* y, int32_t* pos, int BH, int64_t L, int64_t Lp, int D,
                                 rattn_dtype dtype, int cp, int layout, double base, int style,
                                 cudaStream_t stream) {
  RopeArgs a{};
  a.src = static_cast<const uint4*>(x);
  a.dst = static_cast<uint4*>(y);
  a.pos = pos;
  a.BH = BH;
  a.L = static_cast<int>(L);
  a.Lp = static_cast<int>(Lp);
  a.D = D;
  a.c = cp_map_c(Lp, cp, layout);
  a.cp = cp;
  a.layout = layout;
  a.vpr = D * (dtype == RATTN_BF16 ? 2 : 4) / 16;
  a.sign = 1.f;
  a.base = base;
  return dispatch<true>(a, dtype, style, stream);
}

rattn_status launch_unpermute_rope_grad(const void* dy, void* dx, int BH, int64_t L, int64_t Lp, int D,
                                        rattn_dtype dtype, int cp, int layout, double base, int style,
                                        cudaStream_t stream) {
  RopeArgs a{};
  a.src = static_cast<const uint4*>(dy);
  a.dst = static_cast<uint4*>(dx);
  a.pos = nullptr;
  a.BH = BH;
  a.L = static_cast<int>(L);
  a.Lp = static_cast<int>(Lp);
  a.D = D;
  a.c = cp_map_c(Lp, cp, layout);
  a.cp = cp;
  a.layout = layout;
  a.vpr = D * (dtype == RATTN_BF16 ? 2 : 4) / 16;
  a.sign = -1.f;
  a.base = base;
  return dispatch<false>(a, dtype, style, stream);
}

}  // namespace rattn
