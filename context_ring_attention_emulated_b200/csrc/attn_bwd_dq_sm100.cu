// attn_bwd_dq_sm100.cu -- the query gradient of the ring backward as a
// query-stationary pass (sm_100a: tcgen05.mma, TMEM accumulators, TMA-staged
// K/V tiles), for the deterministic mode of the ring backward.
//
// What it computes: the textbook softmax-attention gradient's dQ (the pages
// only call .backward(); [CP-glossary] "Practical use and trade-offs"), over
// the same emulated ring as the forward ([CP-glossary] "How context
// parallelism works"; rank r holds the K/V block of rank (r - t) mod cp at
// hop t):
//   P_ij  = exp(scale q_i.k_j - LSE_i) on visible pairs (LSE saved by the
//           forward), 0 elsewhere,
//   dP    = dO V^T,  dS_ij = P_ij (dP_ij - Delta_i)  (Delta_i = dO_i . O_i),
//   dQ    = scale dS K.
// The key/value-stationary backward adds each key tile's share of dQ into an
// fp32 accumulator from many CTAs at once, in whatever order they arrive. Here
// one CTA owns one 128-row query tile and accumulates its dQ in TMEM over the
// K/V tiles in ring order, so dQ is the same, bit for bit, on every run.
//
// Warp roles (192 threads):
//   warp 0      TMA producer: Q and dO once, then K (3 stages for D = 128)
//               and V (2 stages) tiles of every visible key tile;
//   warp 1      TMEM allocation and tcgen05.mma (the warp waits, one elected lane issues):
//               S_g = Q K_g^T into one of two score buffers, dP_g = dO V_g^T,
//               dQ += dS_g K_g with dS_g read from TMEM; S_{g+2} reuses the
//               buffer once dQ_g (its reader) has completed, dP_{g+1} once the
//               compute warps have read dP_g;
//   warps 2..5  one thread per query row (= TMEM lane): P = exp2(S scale
//               log2 e - LSE log2 e) with the tile's causal / padding /
//               segment mask, dS = P (dP - Delta) packed to bf16 over the
//               first 64 columns of the score buffer; finally dQ x scale
//               rounded once to bf16.
// TMEM columns: S0 [0,128) S1 [128,256) dP [256,384) dQ [384,384+D).
#include <limits.h>
#include <math.h>

#include "debug_check.cuh"
#include "fwd_positions.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace rattn {
namespace {

constexpr int kThreads = 192;
constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // keys per tile
constexpr int kMaxHops = 64;

template <int D>
struct Cfg {
  static constexpr int NSK = (D == 128) ? 3 : 4;  // K stages (K is read by S_g and, later, dQ_g)
  static constexpr int NSV = (D == 128) ? 2 : 4;  // V stages (read by dP_g only)
  static constexpr int TILE = BM * D * 2;
  static constexpr int NBOX = D / 64;
  static constexpr int BOX = BM * 128;
  static constexpr uint32_t T_DP = 256, T_DQ = 384, T_COLS = 512;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = OFF_Q + TILE;
  static constexpr int OFF_K = OFF_DO + TILE;
  static constexpr int OFF_V = OFF_K + NSK * TILE;
  static constexpr int OFF_BAR = OFF_V + NSV * TILE;
  // q_full, K and V full/empty rings, s_full[2], dp_full, dp_free,
  // ds_ready[2], dq_done[2], drain
  static constexpr int NBAR = 1 + 2 * NSK + 2 * NSV + 2 + 1 + 1 + 2 + 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_HOP = (OFF_MISC + 16 + 15) / 16 * 16;  // int4 table
  static constexpr int SMEM = OFF_HOP + kMaxHops * 16 + 1024;        // + alignment slack
  static_assert(OFF_HOP % 16 == 0 && OFF_BAR % 8 == 0, "shared-memory alignment");
  static_assert(SMEM <= 232448, "shared memory budget");
};

struct Params {
  const int32_t* q_pos;
  const int32_t* kv_pos;
  const int32_t* seg;  // packed sequences: segid per slot, or NULL
  const float* lse;    // [BH][nseg*Lq_seg], natural log
  const float* delta;  // [BH][nseg*Lq_seg]
  int BH, group, nseg, Lq_seg, Lk_seg, n_qtiles, causal;
  long long kv_valid;
  float scale, scale_log2;
  __nv_bfloat16* dq;   // [BH][nseg*Lq_seg][D]
  int* err;
  unsigned long long wait_ns;
};

template <int D, bool SEG>  // SEG: packed sequences (segid array present)
__global__ void __launch_bounds__(kThreads, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
              const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sDO = smem + C::OFF_DO;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_q_full = bars;  // Q and dO
  uint64_t* bar_k_full = bars + 1;
  uint64_t* bar_k_empty = bar_k_full + C::NSK;
  uint64_t* bar_v_full = bar_k_empty + C::NSK;
  uint64_t* bar_v_empty = bar_v_full + C::NSV;
  uint64_t* bar_s_full = bar_v_empty + C::NSV;  // [2]
  uint64_t* bar_dp_full = bar_s_full + 2;
  uint64_t* bar_dp_free = bar_dp_full + 1;      // the compute warps have read dP_g
  uint64_t* bar_ds_ready = bar_dp_free + 1;     // [2] dS_g packed in its score buffer
  uint64_t* bar_dq_done = bar_ds_ready + 2;     // [2] dQ += dS_g K_g completed
  uint64_t* bar_drain = bar_dq_done + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  int4* s_hop = reinterpret_cast<int4*>(smem + C::OFF_HOP);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work item: (batch, head) slowest, then rank, then query tile, heaviest first.
  int item = blockIdx.x;
  const int qt = p.n_qtiles - 1 - (item % p.n_qtiles);
  item /= p.n_qtiles;
  const int r = item % p.nseg;
  const int bh = item / p.nseg;
  const int kvh = bh / p.group;
  const int q0 = qt * BM;
  const int q_rows = min(BM, p.Lq_seg - q0);
  const long long q_min = qpos(p, r, q0);
  const long long q_max = qpos(p, r, q0 + q_rows - 1);
  const int nk_tiles = (p.Lk_seg + BN - 1) / BN;

  if (threadIdx.x == 0) {
    mbar_init(bar_q_full, 1);
    for (int i = 0; i < C::NSK; ++i) {
      mbar_init(&bar_k_full[i], 1);
      mbar_init(&bar_k_empty[i], 1);
    }
    for (int i = 0; i < C::NSV; ++i) {
      mbar_init(&bar_v_full[i], 1);
      mbar_init(&bar_v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_s_full[i], 1);
      mbar_init(&bar_ds_ready[i], 4);  // one arrival per compute warp
      mbar_init(&bar_dq_done[i], 1);
    }
    mbar_init(bar_dp_full, 1);
    mbar_init(bar_dp_free, 4);
    mbar_init(bar_drain, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(s_tmem, C::T_COLS);

  // Per hop: visible K/V tiles [first, n_vis) and unmasked ones [f_lo, f_hi),
  // as in the forward (partition points over the non-decreasing positions and
  // segids of a segment; one warp per hop).
  for (int t = warp; t < p.nseg; t += kThreads / 32) {
    const int s = ((r - t) % p.nseg + p.nseg) % p.nseg;
    const int sq_lo = SEG ? segat(p, r, q0) : 0;
    const int sq_hi = SEG ? segat(p, r, q0 + q_rows - 1) : 0;
    const int first = SEG ? warp_partition_point(0, nk_tiles, lane, [&](int m) {
      return segat(p, s, min((m + 1) * BN, p.Lk_seg) - 1) < sq_lo;
    }) : 0;
    const int n_vis = warp_partition_point(first, nk_tiles, lane, [&](int m) {
      const long long kmin = kpos(p, s, m * BN);
      return kmin < p.kv_valid && (!p.causal || kmin <= q_max) && (!SEG || segat(p, s, m * BN) <= sq_hi);
    });
    int f_lo = first, f_hi = first;
    const bool one_seg = !SEG || (sq_lo == sq_hi && (sq_lo & 1) == 0);
    if (one_seg && first < n_vis) {
      int a = first, b = n_vis;
      if (SEG) {
        a = warp_partition_point(first, n_vis, lane, [&](int m) { return segat(p, s, m * BN) < sq_lo; });
        b = warp_partition_point(a, n_vis, lane, [&](int m) {
          return segat(p, s, min((m + 1) * BN, p.Lk_seg) - 1) <= sq_lo;
        });
      }
      f_lo = a;
      f_hi = warp_partition_point(a, b, lane, [&](int m) {
        const bool complete = (m + 1) * BN <= p.Lk_seg;
        const long long kmax = kpos(p, s, min((m + 1) * BN, p.Lk_seg) - 1);
        return complete && kmax < p.kv_valid && (!p.causal || kmax <= q_min);
      });
    }
    if (lane == 0) s_hop[t] = make_int4(first, n_vis, f_lo, f_hi);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  int G = 0;
  for (int t = 0; t < p.nseg; ++t) G += s_hop[t].y - s_hop[t].x;

  int issued_k = 0, issued_v = 0;  // producer bookkeeping for the drain

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && G > 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_do);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      mbar_arrive_expect_tx(bar_q_full, 2 * C::TILE);
      for (int b = 0; b < C::NBOX; ++b) {
        tma_load_4d(sQ + b * C::BOX, &tm_q, bar_q_full, b * 64, q0, r, bh);
        tma_load_4d(sDO + b * C::BOX, &tm_do, bar_q_full, b * 64, q0, r, bh);
      }
      bool ok = true;
      int g = 0;
      for (int t = 0; t < p.nseg && ok; ++t) {
        const int s = ((r - t) % p.nseg + p.nseg) % p.nseg;
        const int nv = s_hop[t].y;
        for (int j = s_hop[t].x; j < nv; ++j, ++g) {
          const int st = g % C::NSK;
          const uint32_t u = g / C::NSK;
          if (u > 0 && !mbar_wait(&bar_k_empty[st], (u - 1) & 1, s_abort, p.wait_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_k_full[st], C::TILE);
          for (int b = 0; b < C::NBOX; ++b)
            tma_load_4d(sK + st * C::TILE + b * C::BOX, &tm_k, &bar_k_full[st], b * 64, j * BN, s, kvh);
          ++issued_k;
          const int sv = g % C::NSV;
          const uint32_t uv = g / C::NSV;
          if (uv > 0 && !mbar_wait(&bar_v_empty[sv], (uv - 1) & 1, s_abort, p.wait_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_v_full[sv], C::TILE);
          for (int b = 0; b < C::NBOX; ++b)
            tma_load_4d(sV + sv * C::TILE + b * C::BOX, &tm_v, &bar_v_full[sv], b * 64, j * BN, s, kvh);
          ++issued_v;
        }
      }
      if (!ok) record_failure(s_abort, p.err, SITE_BWD_LOAD);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issue
    if (G > 0) {  // the whole warp walks the schedule and waits; one elected lane issues
      const uint32_t idesc_s = idesc_bf16_f32(BM, BN, 0, 0);
      const uint32_t idesc_q = idesc_bf16_f32(BM, D, 0, 1);
      const uint32_t sQa = smem_u32(sQ), sDOa = smem_u32(sDO);
      bool ok = warp_wait(bar_q_full, 0, s_abort, p.wait_ns);
      // A x B^T over D for 128 x 128 tiles, both operands K-major in smem
      auto mma_nt = [&](uint32_t d, uint32_t a, uint32_t b) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
          umma_ss(d, sdesc_sw128(a + off, 16, 1024), sdesc_sw128(b + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      // S_g = Q K_g^T into score buffer g % 2
      auto issue_s = [&](int g) -> bool {
        const int st = g % C::NSK;
        if (!warp_wait(&bar_k_full[st], (g / C::NSK) & 1, s_abort, p.wait_ns)) return false;
        tc_fence_after();
        if (elect_one()) {
          mma_nt(tmem + (g & 1) * 128, sQa, smem_u32(sK + st * C::TILE));
          umma_commit(&bar_s_full[g & 1]);
        }
        __syncwarp();
        return true;
      };
      // dP_g = dO V_g^T
      auto issue_dp = [&](int g) -> bool {
        const int sv = g % C::NSV;
        if (!warp_wait(&bar_v_full[sv], (g / C::NSV) & 1, s_abort, p.wait_ns)) return false;
        tc_fence_after();
        if (elect_one()) {
          mma_nt(tmem + C::T_DP, sDOa, smem_u32(sV + sv * C::TILE));
          umma_commit(bar_dp_full);
          umma_commit(&bar_v_empty[sv]);
        }
        __syncwarp();
        return true;
      };
      // Per tile g: dP_{g+1} as soon as the compute warps have read dP_g (it
      // runs while they form dS_g), then dQ += dS_g K_g, then S_{g+2} into
      // dS_g's buffer once dQ_g has read it.
      if (ok) ok = issue_s(0) && issue_dp(0);
      if (ok && G > 1) ok = issue_s(1);
      for (int g = 0; g < G && ok; ++g) {
        if (g + 1 < G) {
          ok = warp_wait(bar_dp_free, g & 1, s_abort, p.wait_ns) && issue_dp(g + 1);
          if (!ok) break;
        }
        // dQ += dS_g K_g: dS_g (bf16, 128 query rows x 128 keys) from the
        // first 64 columns of its score buffer, K_g as an MN-major B operand
        ok = warp_wait(&bar_ds_ready[g & 1], (g >> 1) & 1, s_abort, p.wait_ns);
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
          const int st = g % C::NSK;
          const uint32_t sKa = smem_u32(sK + st * C::TILE);
          const uint32_t a_t = tmem + (g & 1) * 128;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint64_t bd = sdesc_sw128(sKa + kk * 2048, C::BOX, 1024);
            umma_ts(tmem + C::T_DQ, a_t + kk * 8, bd, idesc_q, (g > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bar_dq_done[g & 1]);
          umma_commit(&bar_k_empty[st]);
        }
        __syncwarp();
        if (g + 2 < G)
          ok = warp_wait(&bar_dq_done[g & 1], (g >> 1) & 1, s_abort, p.wait_ns) && issue_s(g + 2);
      }
      if (!ok && lane == 0) record_failure(s_abort, p.err, SITE_BWD_MMA);
    }
  } else {
    // ------------------------------------------------ dS and the epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const bool row_valid = row < q_rows;
    const long long grow = (static_cast<long long>(bh) * p.nseg + r) * p.Lq_seg + q0 + row;  // row of lse/delta/dq
    const bool grow_ok = row_valid && in_bounds(grow, static_cast<long long>(p.BH) * p.nseg * p.Lq_seg, p.err, 21);
    const long long my_pos = row_valid ? qpos(p, r, q0 + row) : q_max;
    const int my_seg = (SEG && row_valid) ? segat(p, r, q0 + row) : 1;  // odd: sees nothing
    // P = exp2(S scale log2 e - LSE log2 e); a row without a visible key
    // (LSE = -inf) and a padding row get P = 0 through an infinite offset.
    float lse2 = INFINITY, dlt = 0.f;
    if (grow_ok) {
      const float l = __ldg(p.lse + grow);
      lse2 = (l == -INFINITY) ? INFINITY : l * 1.4426950408889634f;
      dlt = __ldg(p.delta + grow);
    }
    const float sl2 = p.scale_log2;
    bool ok = true;
    int g = 0;
    for (int t = 0; t < p.nseg && ok; ++t) {
      const int s = ((r - t) % p.nseg + p.nseg) % p.nseg;
      const int nv = s_hop[t].y, f_lo = s_hop[t].z, f_hi = s_hop[t].w;
      for (int j = s_hop[t].x; j < nv; ++j, ++g) {
        // Visible keys of this row in the tile: [klo, khi) (all of it when
        // unmasked), found as in the forward for masked tiles.
        int klo = 0, khi = BN;
        if (j < f_lo || j >= f_hi) {
          const int n = min(BN, p.Lk_seg - j * BN);
          const long long kbase = static_cast<long long>(s) * p.Lk_seg + j * BN;
          int kp4[4], ks4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int idx = 4 * lane + e;
            const bool inb = idx < n && in_bounds(kbase + idx, static_cast<long long>(p.nseg) * p.Lk_seg, p.err, 22);
            kp4[e] = inb ? (p.kv_pos ? __ldg(p.kv_pos + kbase + idx) : j * BN + idx) : INT_MAX;
            ks4[e] = (SEG && inb) ? __ldg(p.seg + kbase + idx) : INT_MAX;
          }
          if (SEG) {
            int lo = 0, hi = n;
#pragma unroll 1
            for (int step = 0; step < 8; ++step) {
              const int mid = (lo + hi) >> 1;
              const int sg = warp_elem128(ks4, mid);
              if (lo < hi) {
                if (sg >= my_seg) hi = mid; else lo = mid + 1;
              }
            }
            klo = (my_seg & 1) ? n : lo;
          }
          int lo = klo, hi = n;
#pragma unroll 1
          for (int step = 0; step < 8; ++step) {
            const int mid = (lo + hi) >> 1;
            const long long kp = warp_elem128(kp4, mid);
            const int sg = SEG ? warp_elem128(ks4, mid) : 0;
            const bool vis = kp < p.kv_valid && (!p.causal || kp <= my_pos) && (!SEG || sg == my_seg);
            if (lo < hi) {
              if (vis) lo = mid + 1; else hi = mid;
            }
          }
          khi = lo;
        }
        if (!warp_wait(&bar_s_full[g & 1], (g >> 1) & 1, s_abort, p.wait_ns) ||
            !warp_wait(bar_dp_full, g & 1, s_abort, p.wait_ns)) {
          record_failure(s_abort, p.err, SITE_BWD_COMPUTE);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t s_addr = tmem + lane_base + (g & 1) * 128;
        const uint32_t dp_addr = tmem + lane_base + C::T_DP;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t sv[2][32], dv[2][32];
          tmem_ld32(s_addr + h * 64, sv[0]);
          tmem_ld32(s_addr + h * 64 + 32, sv[1]);
          tmem_ld32(dp_addr + h * 64, dv[0]);
          tmem_ld32(dp_addr + h * 64 + 32, dv[1]);
          tmem_wait_ld();
          if (h == 1) {  // dP_g is in registers: the next dP may overwrite it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_dp_free);
          }
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int c0 = h * 64 + 2 * i;
            const float sa = __uint_as_float(sv[(2 * i) >> 5][(2 * i) & 31]);
            const float sb = __uint_as_float(sv[(2 * i + 1) >> 5][(2 * i + 1) & 31]);
            const float pa = (c0 >= klo && c0 < khi) ? ex2_approx(fmaf(sa, sl2, -lse2)) : 0.f;
            const float pb = (c0 + 1 >= klo && c0 + 1 < khi) ? ex2_approx(fmaf(sb, sl2, -lse2)) : 0.f;
            const float da = pa * (__uint_as_float(dv[(2 * i) >> 5][(2 * i) & 31]) - dlt);
            const float db = pb * (__uint_as_float(dv[(2 * i + 1) >> 5][(2 * i + 1) & 31]) - dlt);
            pk[i] = pack_bf16x2(da, db);
          }
          tmem_st32(s_addr + h * 32, pk);  // dS over the scores already read
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_ds_ready[g & 1]);  // one arrival per warp
      }
    }

    // ---------------------------------------------------------- epilogue
    if (ok && G > 0) {
      if (!warp_wait(&bar_dq_done[(G - 1) & 1], ((G - 1) >> 1) & 1, s_abort, p.wait_ns)) {
        record_failure(s_abort, p.err, SITE_BWD_EPILOGUE);
        ok = false;
      }
    }
    if (ok) {
      if (G > 0) tc_fence_after();
      const uint32_t q_addr = tmem + lane_base + C::T_DQ;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        if (G > 0) {
          tmem_ld32(q_addr + c * 32, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0u;
        }
        if (grow_ok) {
          uint4* dst = reinterpret_cast<uint4*>(p.dq + grow * D + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(v[8 * i + 0]) * p.scale, __uint_as_float(v[8 * i + 1]) * p.scale);
            w.y = pack_bf16x2(__uint_as_float(v[8 * i + 2]) * p.scale, __uint_as_float(v[8 * i + 3]) * p.scale);
            w.z = pack_bf16x2(__uint_as_float(v[8 * i + 4]) * p.scale, __uint_as_float(v[8 * i + 5]) * p.scale);
            w.w = pack_bf16x2(__uint_as_float(v[8 * i + 6]) * p.scale, __uint_as_float(v[8 * i + 7]) * p.scale);
            dst[i] = w;
          }
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  if (warp == 0 && lane == 0 && G > 0) {
    drain_wait(bar_q_full, 0);
    for (int g = max(0, issued_k - C::NSK); g < issued_k; ++g)
      drain_wait(&bar_k_full[g % C::NSK], (g / C::NSK) & 1);
    for (int g = max(0, issued_v - C::NSV); g < issued_v; ++g)
      drain_wait(&bar_v_full[g % C::NSV], (g / C::NSV) & 1);
  }
  if (warp == 1 && G > 0) {  // the lane that issued the products commits
    if (elect_one()) {
      umma_commit(bar_drain);
      if (!drain_wait(bar_drain, 0)) record_failure(s_abort, p.err, SITE_DRAIN);
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::T_COLS);
  }
}

template <int D>
rattn_status launch(const BwdArgs& a, const DevCtx& ctx, bool run) {
  using C = Cfg<D>;
  if (a.Lseg > INT32_MAX - BM || a.nseg > kMaxHops) return RATTN_ERR_UNSUPPORTED;
  if (a.group < 1 || a.BH % a.group) return RATTN_ERR_INVALID_ARG;
  const int n_qtiles = static_cast<int>((a.Lseg + BM - 1) / BM);
  const long long grid = static_cast<long long>(a.BH) * a.nseg * n_qtiles;
  if (grid == 0) return RATTN_OK;
  if (grid > INT32_MAX) return RATTN_ERR_UNSUPPORTED;
  CUtensorMap tq, tdo, tk, tv;
  rattn_status st;
  if ((st = make_tmap_bf16(&tq, a.q, D, a.Lseg, a.nseg, a.BH, BM)) != RATTN_OK) return st;
  if ((st = make_tmap_bf16(&tdo, a.dout, D, a.Lseg, a.nseg, a.BH, BM)) != RATTN_OK) return st;
  if ((st = make_tmap_bf16(&tk, a.k, D, a.Lseg, a.nseg, a.BH / a.group, BN)) != RATTN_OK) return st;
  if ((st = make_tmap_bf16(&tv, a.v, D, a.Lseg, a.nseg, a.BH / a.group, BN)) != RATTN_OK) return st;
  const void* kfn = a.seg ? reinterpret_cast<const void*>(&dq_kernel<D, true>)
                         : reinterpret_cast<const void*>(&dq_kernel<D, false>);
  if ((st = set_smem_attr(kfn, C::SMEM)) != RATTN_OK) return st;
  if (!run) return RATTN_OK;
  Params p;
  p.q_pos = a.pos;
  p.kv_pos = a.pos;
  p.seg = a.seg;
  p.lse = a.lse;
  p.delta = a.delta;
  p.BH = a.BH;
  p.group = a.group;
  p.nseg = a.nseg;
  p.Lq_seg = static_cast<int>(a.Lseg);
  p.Lk_seg = static_cast<int>(a.Lseg);
  p.n_qtiles = n_qtiles;
  p.causal = a.causal;
  p.kv_valid = a.kv_valid;
  p.scale = a.scale;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.dq = static_cast<__nv_bfloat16*>(a.dq);
  p.err = ctx.err_word;
  p.wait_ns = ctx.wait_ns;
  if (a.seg)
    dq_kernel<D, true><<<static_cast<unsigned>(grid), kThreads, C::SMEM, a.stream>>>(tq, tdo, tk, tv, p);
  else
    dq_kernel<D, false><<<static_cast<unsigned>(grid), kThreads, C::SMEM, a.stream>>>(tq, tdo, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? RATTN_OK : RATTN_ERR_CUDA;
}

}  // namespace

rattn_status launch_bwd_dq_sm100(const BwdArgs& a, const DevCtx& ctx, bool run) {
  if (a.dtype != RATTN_BF16) return RATTN_ERR_UNSUPPORTED;
  if (a.D == 128) return launch<128>(a, ctx, run);
  if (a.D == 64) return launch<64>(a, ctx, run);
  return RATTN_ERR_UNSUPPORTED;
}

}  // namespace rattn
