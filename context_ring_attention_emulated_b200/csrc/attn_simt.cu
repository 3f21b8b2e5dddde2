// attn_simt.cu -- exact-fp32 ring / partial attention (forward and backward)
// on the CUDA cores, for fp32 inputs.
//
// Same method as the tensor-core path ([CP-glossary] "How context
// parallelism works", [Ring-page] "Technical insight"): each query row keeps a
// running max m, running normaliser l and an unnormalised accumulator, and
// folds the keys of every hop in ring order (hop t of rank r holds the block
// of rank (r - t) mod nseg), rescaling the accumulator whenever m grows.
// fp32 FMA only (no TF32), one thread per query row, K/V tiles staged in
// shared memory. The backward pass recomputes P from the saved LSE:
//   P = exp(scale q.k - LSE), dV_j += P dO_i, dP = dO_i.v_j,
//   dS = P (dP - Delta_i), dQ_i += scale dS k_j, dK_j += scale dS q_i,
// with Delta_i = dO_i . O_i.
#include <climits>
#include <math.h>

#include "internal.h"

namespace rattn {
namespace {

constexpr int kRows = 64;   // query (or key) rows per CTA, one per thread
constexpr int kTile = 32;   // staged rows per shared-memory tile

struct SimtFwd {
  const float* q;
  const float* k;
  const float* v;
  const int32_t* q_pos;
  const int32_t* kv_pos;
  const int32_t* seg;  // packed sequences: segid per slot (q and kv share it), or NULL
  int BH, group, nseg, Lq_seg, Lk_seg, D, causal;
  long long kv_valid;
  float scale;
  float* o;
  float* lse;
};

__device__ __forceinline__ long long pos_at(const int32_t* pos, long long base, int row) {
  return pos ? static_cast<long long>(pos[base + row]) : row;
}

// Packed sequences: a key is visible only to queries with the same even segid.
__device__ __forceinline__ bool seg_ok(const int32_t* seg, long long qi, long long ki) {
  if (!seg) return true;
  const int sk = seg[ki];
  return sk == seg[qi] && (sk & 1) == 0;
}

template <int DMAX>
__global__ void __launch_bounds__(kRows) fwd_simt_kernel(const SimtFwd p) {
  __shared__ float sk[kTile][DMAX];
  __shared__ float sv[kTile][DMAX];
  __shared__ long long skp[kTile];
  __shared__ int sks[kTile];
  const int nqt = (p.Lq_seg + kRows - 1) / kRows;
  int item = blockIdx.x;
  const int qt = item % nqt;
  item /= nqt;
  const int r = item % p.nseg;
  const int bh = item / p.nseg;
  const int row = qt * kRows + threadIdx.x;
  const bool valid = row < p.Lq_seg;
  const long long qbase = (static_cast<long long>(bh) * p.nseg + r) * p.Lq_seg;
  const int my_seg = p.seg ? p.seg[static_cast<long long>(r) * p.Lq_seg + (valid ? row : 0)] : 0;
  const int last_row = min(qt * kRows + kRows, p.Lq_seg) - 1;
  const long long my_pos = pos_at(p.q_pos, static_cast<long long>(r) * p.Lq_seg, valid ? row : last_row);
  const long long blk_max = pos_at(p.q_pos, static_cast<long long>(r) * p.Lq_seg, last_row);

  float qr[DMAX], acc[DMAX];
#pragma unroll
  for (int d = 0; d < DMAX; ++d) {
    qr[d] = (valid && d < p.D) ? p.q[(qbase + row) * p.D + d] : 0.f;
    acc[d] = 0.f;
  }
  float m = -INFINITY, l = 0.f;

  for (int t = 0; t < p.nseg; ++t) {
    const int s = ((r - t) % p.nseg + p.nseg) % p.nseg;
    const long long kbase = (static_cast<long long>(bh / p.group) * p.nseg + s) * p.Lk_seg;
    for (int k0 = 0; k0 < p.Lk_seg; k0 += kTile) {
      const long long first = pos_at(p.kv_pos, static_cast<long long>(s) * p.Lk_seg, k0);
      if (first >= p.kv_valid || (p.causal && first > blk_max)) break;  // positions are non-decreasing
      const int n = min(kTile, p.Lk_seg - k0);
      __syncthreads();
      for (int e = threadIdx.x; e < kTile * DMAX; e += kRows) {
        const int kr = e / DMAX, d = e % DMAX;
        const bool in = kr < n && d < p.D;
        sk[kr][d] = in ? p.k[(kbase + k0 + kr) * p.D + d] : 0.f;
        sv[kr][d] = in ? p.v[(kbase + k0 + kr) * p.D + d] : 0.f;
      }
      for (int kr = threadIdx.x; kr < kTile; kr += kRows) {
        skp[kr] = kr < n ? pos_at(p.kv_pos, static_cast<long long>(s) * p.Lk_seg, k0 + kr) : LLONG_MAX;
        sks[kr] = (kr < n && p.seg) ? p.seg[static_cast<long long>(s) * p.Lk_seg + k0 + kr] : 0;
      }
      __syncthreads();
      for (int kr = 0; kr < n; ++kr) {
        const long long kp = skp[kr];
        if (kp >= p.kv_valid || (p.causal && kp > my_pos)) continue;
        if (p.seg && (sks[kr] != my_seg || (my_seg & 1))) continue;
        float x = 0.f;
#pragma unroll
        for (int d = 0; d < DMAX; ++d) x = fmaf(qr[d], sk[kr][d], x);
        x *= p.scale;
        if (x > m) {
          const float alpha = expf(m - x);  // m = -inf gives 0
          l *= alpha;
#pragma unroll
          for (int d = 0; d < DMAX; ++d) acc[d] *= alpha;
          m = x;
        }
        const float w = expf(x - m);
        l += w;
#pragma unroll
        for (int d = 0; d < DMAX; ++d) acc[d] = fmaf(w, sv[kr][d], acc[d]);
      }
    }
  }
  if (valid) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
    for (int d = 0; d < p.D; ++d) p.o[(qbase + row) * p.D + d] = acc[d] * inv;
    p.lse[qbase + row] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}

// ----------------------------------------------------------------- backward

struct SimtBwd {
  const float* q;
  const float* k;
  const float* v;
  const float* o;
  const float* dout;
  const float* lse;
  const int32_t* pos;
  const int32_t* seg;  // packed sequences: segid per slot, or NULL
  int BH, group, nseg, Lseg, D, causal;
  long long kv_valid;
  float scale;
  float* dq;
  float* dk;
  float* dv;
  float* delta;
};

__global__ void delta_simt_kernel(const SimtBwd p, long long rows) {
  const long long rr = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  if (rr >= rows) return;
  float s = 0.f;
  for (int d = 0; d < p.D; ++d) s = fmaf(p.o[rr * p.D + d], p.dout[rr * p.D + d], s);
  p.delta[rr] = s;
}

// One thread per query row: dQ_i = scale * sum_j P_ij (dP_ij - Delta_i) k_j.
template <int DMAX>
__global__ void __launch_bounds__(kRows) dq_simt_kernel(const SimtBwd p) {
  __shared__ float sk[kTile][DMAX];
  __shared__ float sv[kTile][DMAX];
  __shared__ long long skp[kTile];
  const int nqt = (p.Lseg + kRows - 1) / kRows;
  int item = blockIdx.x;
  const int qt = item % nqt;
  item /= nqt;
  const int r = item % p.nseg;
  const int bh = item / p.nseg;
  const int row = qt * kRows + threadIdx.x;
  const bool valid = row < p.Lseg;
  const long long qbase = (static_cast<long long>(bh) * p.nseg + r) * p.Lseg;
  const int last_row = min(qt * kRows + kRows, p.Lseg) - 1;
  const long long my_pos = p.pos[static_cast<long long>(r) * p.Lseg + (valid ? row : last_row)];
  const long long blk_max = p.pos[static_cast<long long>(r) * p.Lseg + last_row];
  const long long my_slot = static_cast<long long>(r) * p.Lseg + (valid ? row : last_row);
  float qr[DMAX], dor[DMAX], g[DMAX];
#pragma unroll
  for (int d = 0; d < DMAX; ++d) {
    qr[d] = (valid && d < p.D) ? p.q[(qbase + row) * p.D + d] : 0.f;
    dor[d] = (valid && d < p.D) ? p.dout[(qbase + row) * p.D + d] : 0.f;
    g[d] = 0.f;
  }
  const float lse = valid ? p.lse[qbase + row] : 0.f;
  const float dl = valid ? p.delta[qbase + row] : 0.f;
  for (int t = 0; t < p.nseg; ++t) {
    const int s = ((r - t) % p.nseg + p.nseg) % p.nseg;
    const long long kbase = (static_cast<long long>(bh / p.group) * p.nseg + s) * p.Lseg;
    for (int k0 = 0; k0 < p.Lseg; k0 += kTile) {
      const long long first = p.pos[static_cast<long long>(s) * p.Lseg + k0];
      if (first >= p.kv_valid || (p.causal && first > blk_max)) break;
      const int n = min(kTile, p.Lseg - k0);
      __syncthreads();
      for (int e = threadIdx.x; e < kTile * DMAX; e += kRows) {
        const int kr = e / DMAX, d = e % DMAX;
        const bool in = kr < n && d < p.D;
        sk[kr][d] = in ? p.k[(kbase + k0 + kr) * p.D + d] : 0.f;
        sv[kr][d] = in ? p.v[(kbase + k0 + kr) * p.D + d] : 0.f;
      }
      for (int kr = threadIdx.x; kr < kTile; kr += kRows)
        skp[kr] = kr < n ? p.pos[static_cast<long long>(s) * p.Lseg + k0 + kr] : LLONG_MAX;
      __syncthreads();
      if (!valid) continue;
      for (int kr = 0; kr < n; ++kr) {
        const long long kp = skp[kr];
        if (kp >= p.kv_valid || (p.causal && kp > my_pos)) continue;
        if (!seg_ok(p.seg, my_slot, static_cast<long long>(s) * p.Lseg + k0 + kr)) continue;
        float x = 0.f, dp = 0.f;
#pragma unroll
        for (int d = 0; d < DMAX; ++d) {
          x = fmaf(qr[d], sk[kr][d], x);
          dp = fmaf(dor[d], sv[kr][d], dp);
        }
        const float pr = expf(x * p.scale - lse);
        const float ds = pr * (dp - dl);
#pragma unroll
        for (int d = 0; d < DMAX; ++d) g[d] = fmaf(ds, sk[kr][d], g[d]);
      }
    }
  }
  if (valid)
    for (int d = 0; d < p.D; ++d) p.dq[(qbase + row) * p.D + d] = g[d] * p.scale;
}

// One thread per key row: dV_j = sum_i P_ij dO_i, dK_j = scale sum_i dS_ij q_i,
// over the queries of every rank (the K/V block visits every rank's Q) and of
// every query head of the key/value head's group.
template <int DMAX>
__global__ void __launch_bounds__(kRows) dkdv_simt_kernel(const SimtBwd p) {
  __shared__ float sq[kTile][DMAX];
  __shared__ float sdo[kTile][DMAX];
  __shared__ float slse[kTile], sdl[kTile];
  __shared__ long long sqp[kTile];
  const int nkt = (p.Lseg + kRows - 1) / kRows;
  int item = blockIdx.x;
  const int kt = item % nkt;
  item /= nkt;
  const int s = item % p.nseg;
  const int kvh = item / p.nseg;  // (batch, key/value head)
  const int row = kt * kRows + threadIdx.x;
  const bool valid = row < p.Lseg;
  const long long kbase = (static_cast<long long>(kvh) * p.nseg + s) * p.Lseg;
  const int first_row = kt * kRows;
  const long long my_pos = p.pos[static_cast<long long>(s) * p.Lseg + (valid ? row : first_row)];
  const long long blk_min = p.pos[static_cast<long long>(s) * p.Lseg + first_row];
  const bool key_live = valid && my_pos < p.kv_valid;
  const long long my_slot = static_cast<long long>(s) * p.Lseg + (valid ? row : first_row);
  float kr_[DMAX], vr[DMAX], gk[DMAX], gv[DMAX];
#pragma unroll
  for (int d = 0; d < DMAX; ++d) {
    kr_[d] = (valid && d < p.D) ? p.k[(kbase + row) * p.D + d] : 0.f;
    vr[d] = (valid && d < p.D) ? p.v[(kbase + row) * p.D + d] : 0.f;
    gk[d] = 0.f;
    gv[d] = 0.f;
  }
  for (int hr = 0; hr < p.group * p.nseg; ++hr) {
    const int r = hr % p.nseg;
    const long long qbase = (static_cast<long long>(kvh * p.group + hr / p.nseg) * p.nseg + r) * p.Lseg;
    for (int q0 = 0; q0 < p.Lseg; q0 += kTile) {
      const int n = min(kTile, p.Lseg - q0);
      const long long last = p.pos[static_cast<long long>(r) * p.Lseg + q0 + n - 1];
      if (p.causal && last < blk_min) continue;  // no query of this tile sees this key block
      __syncthreads();
      for (int e = threadIdx.x; e < kTile * DMAX; e += kRows) {
        const int qr = e / DMAX, d = e % DMAX;
        const bool in = qr < n && d < p.D;
        sq[qr][d] = in ? p.q[(qbase + q0 + qr) * p.D + d] : 0.f;
        sdo[qr][d] = in ? p.dout[(qbase + q0 + qr) * p.D + d] : 0.f;
      }
      for (int qr = threadIdx.x; qr < kTile; qr += kRows) {
        sqp[qr] = qr < n ? p.pos[static_cast<long long>(r) * p.Lseg + q0 + qr] : LLONG_MIN;
        slse[qr] = qr < n ? p.lse[qbase + q0 + qr] : 0.f;
        sdl[qr] = qr < n ? p.delta[qbase + q0 + qr] : 0.f;
      }
      __syncthreads();
      if (!key_live) continue;
      for (int qr = 0; qr < n; ++qr) {
        if (p.causal && my_pos > sqp[qr]) continue;
        if (!seg_ok(p.seg, static_cast<long long>(r) * p.Lseg + q0 + qr, my_slot)) continue;
        float x = 0.f, dp = 0.f;
#pragma unroll
        for (int d = 0; d < DMAX; ++d) {
          x = fmaf(sq[qr][d], kr_[d], x);
          dp = fmaf(sdo[qr][d], vr[d], dp);
        }
        const float pr = expf(x * p.scale - slse[qr]);
        const float ds = pr * (dp - sdl[qr]);
#pragma unroll
        for (int d = 0; d < DMAX; ++d) {
          gv[d] = fmaf(pr, sdo[qr][d], gv[d]);
          gk[d] = fmaf(ds, sq[qr][d], gk[d]);
        }
      }
    }
  }
  if (valid) {
    for (int d = 0; d < p.D; ++d) {
      p.dk[(kbase + row) * p.D + d] = gk[d] * p.scale;
      p.dv[(kbase + row) * p.D + d] = gv[d];
    }
  }
}

template <int DMAX>
rattn_status fwd_launch(const SimtFwd& p, cudaStream_t stream) {
  const long long nqt = (p.Lq_seg + kRows - 1) / kRows;
  const long long grid = static_cast<long long>(p.BH) * p.nseg * nqt;
  if (grid == 0) return RATTN_OK;
  if (grid > INT32_MAX) return RATTN_ERR_UNSUPPORTED;
  fwd_simt_kernel<DMAX><<<static_cast<unsigned>(grid), kRows, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? RATTN_OK : RATTN_ERR_CUDA;
}

template <int DMAX>
rattn_status bwd_launch(const SimtBwd& p, cudaStream_t stream) {
  const long long rows = static_cast<long long>(p.BH) * p.nseg * p.Lseg;
  const long long nt = (p.Lseg + kRows - 1) / kRows;
  const long long grid = static_cast<long long>(p.BH) * p.nseg * nt;
  if (grid == 0) return RATTN_OK;
  if (grid > INT32_MAX) return RATTN_ERR_UNSUPPORTED;
  delta_simt_kernel<<<static_cast<unsigned>((rows + 255) / 256), 256, 0, stream>>>(p, rows);
  dq_simt_kernel<DMAX><<<static_cast<unsigned>(grid), kRows, 0, stream>>>(p);
  dkdv_simt_kernel<DMAX><<<static_cast<unsigned>(grid / p.group), kRows, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? RATTN_OK : RATTN_ERR_CUDA;
}

}  // namespace

rattn_status launch_fwd_simt(const FwdArgs& a) {
  if (a.dtype != RATTN_F32 || a.D > 128 || a.D % 4) return RATTN_ERR_UNSUPPORTED;
  if (a.group < 1 || a.BH % a.group) return RATTN_ERR_INVALID_ARG;
  if (a.Lq_seg > INT32_MAX - kRows || a.Lk_seg > INT32_MAX - kTile) return RATTN_ERR_UNSUPPORTED;
  SimtFwd p;
  p.q = static_cast<const float*>(a.q);
  p.k = static_cast<const float*>(a.k);
  p.v = static_cast<const float*>(a.v);
  p.q_pos = a.q_pos;
  p.kv_pos = a.kv_pos;
  p.seg = a.seg;
  p.BH = a.BH;
  p.group = a.group;
  p.nseg = a.nseg;
  p.Lq_seg = static_cast<int>(a.Lq_seg);
  p.Lk_seg = static_cast<int>(a.Lk_seg);
  p.D = a.D;
  p.causal = a.causal;
  p.kv_valid = a.kv_valid;
  p.scale = a.scale;
  p.o = static_cast<float*>(a.o);
  p.lse = a.lse;
  if (a.D <= 32) return fwd_launch<32>(p, a.stream);
  if (a.D <= 64) return fwd_launch<64>(p, a.stream);
  return fwd_launch<128>(p, a.stream);
}

rattn_status launch_bwd_simt(const BwdArgs& a) {
  if (a.dtype != RATTN_F32 || a.D > 128 || a.D % 4) return RATTN_ERR_UNSUPPORTED;
  if (a.group < 1 || a.BH % a.group) return RATTN_ERR_INVALID_ARG;
  if (a.Lseg > INT32_MAX - kRows) return RATTN_ERR_UNSUPPORTED;
  SimtBwd p;
  p.q = static_cast<const float*>(a.q);
  p.k = static_cast<const float*>(a.k);
  p.v = static_cast<const float*>(a.v);
  p.o = static_cast<const float*>(a.o);
  p.dout = static_cast<const float*>(a.dout);
  p.lse = a.lse;
  p.pos = a.pos;
  p.seg = a.seg;
  p.BH = a.BH;
  p.group = a.group;
  p.nseg = a.nseg;
  p.Lseg = static_cast<int>(a.Lseg);
  p.D = a.D;
  p.causal = a.causal;
  p.kv_valid = a.kv_valid;
  p.scale = a.scale;
  p.dq = static_cast<float*>(a.dq);
  p.dk = static_cast<float*>(a.dk);
  p.dv = static_cast<float*>(a.dv);
  p.delta = a.delta;
  if (a.D <= 32) return bwd_launch<32>(p, a.stream);
  if (a.D <= 64) return bwd_launch<64>(p, a.stream);
  return bwd_launch<128>(p, a.stream);
}

}  // namespace rattn
