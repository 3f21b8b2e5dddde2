// attn_fwd_wide_sm100.cu -- the ring / partial attention forward with 256-key
// tiles (sm_100a: tcgen05.mma, TMEM accumulators, TMA-staged K/V tiles).
//
// What it computes ([CP-glossary] "How context parallelism works";
// [Ring-page] "Deep dive", "Technical insight"): every emulated rank keeps its
// query tile fixed while the K/V blocks of the ring arrive hop by hop (rank r
// holds the block of rank (r - t) mod cp at hop t); each block's scores are
// folded into a running row max and normaliser, earlier sums rescaled when the
// max grows, so the result equals full softmax attention. Tiles that the
// causal position relation fully masks are skipped.
//
// Why 256-key tiles: the score product S = Q K^T is issued as N = 256 MMAs
// (256 keys at once), half as many instructions per FLOP as N = 128, which
// leaves the issuing warp more slack per product. The TMEM plan keeps one 256-column
// score buffer, a separate 128-column buffer for P (bf16, 256 keys packed two
// per column) and O: S [0,256) P [256,384) O [384,512). Because P does not
// overwrite the scores, the next tile's score product may start as soon as the
// softmax warps have read the scores into registers, and runs while they work.
//
// One CTA owns one 128-row query tile of one (batch, head, rank). Warp roles
// (384 threads):
//   warp 8      TMA producer: Q once, K tiles (256 x D) through 2 stages, each
//               V tile (256 x D) into its one stage one tile behind the K
//               loads (so a K load never queues behind a V stage that frees
//               late);
//   warp 9      TMEM allocation and tcgen05.mma (the whole warp waits, one
//               lane chosen by elect.sync issues), in the order
//               S_{g+1} (once the scores S_g are read), PV_g (once P_g is in
//               TMEM);
//   warps 0..7  softmax, two warps per TMEM lane quarter: warp half h takes
//               keys [128 h, 128 h + 128) of every tile and output columns
//               [h D/2, (h+1) D/2). P_g is first formed against the reference
//               max kept so far, without a row max; the two warps of a pair
//               then meet at a named barrier (bar.red.or) and, only if a row
//               of either half needs a new reference (its first visible keys,
//               or a half-row sum above 2^16), combine their row maxima through
//               shared memory, rescale lazily and form P_g again. Both leave
//               together on any failure, so neither can be left waiting; row
//               sums are added once at the end. P_g is written only after
//               PV_{g-1}, the last reader of the P buffer, has completed.
//   warps 10-11 idle (they complete the producer / MMA warpgroup, whose
//               registers go to the softmax warpgroups by setmaxnreg).
#include <limits.h>
#include <math.h>

#include "debug_check.cuh"
#include "fwd_positions.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace rattn {
namespace {

constexpr int kThreads = 384;
// Registers: launched at kLaunchRegs (12 warps); the producer / MMA warpgroup
// (warps 8..11) shrinks to kRegsLoad so that each softmax warpgroup can hold
// 128 scores per thread (kRegsSoftmax).
constexpr int kLaunchRegs = 168;
constexpr int kRegsLoad = 56;
constexpr int kRegsSoftmax = 224;
static_assert(kRegsLoad + 2 * kRegsSoftmax == 3 * kLaunchRegs, "register split must balance");
constexpr int BM = 128;  // query rows per tile
constexpr int BN = 256;  // keys per tile
constexpr int D = 128;   // head dimension of this kernel
constexpr int kMaxHops = 32;

struct Cfg {
  static constexpr int NSK = 2;                  // K stages
  static constexpr int QTILE = BM * D * 2;       // 32 KB, two 128-row boxes
  static constexpr int QBOX = BM * 128;          // 16 KB
  static constexpr int KTILE = BN * D * 2;       // 64 KB, two 256-row boxes
  static constexpr int KBOX = BN * 128;          // 32 KB
  static constexpr uint32_t T_P = 256, T_O = 384, T_COLS = 512;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QTILE;
  static constexpr int OFF_V = OFF_K + NSK * KTILE;
  static constexpr int OFF_BAR = OFF_V + KTILE;
  // q_full, k_full[2], k_empty[2], v_full, v_empty, s_full, s_free, p_ready,
  // o_done, drain
  static constexpr int NBAR = 1 + 2 * NSK + 2 + 4 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_HOP = (OFF_MISC + 16 + 15) / 16 * 16;  // int4 table
  static constexpr int OFF_XCH = OFF_HOP + kMaxHops * 16;           // float [parity][half][row]
  static constexpr int SMEM = OFF_XCH + 2 * 2 * BM * 4;
  static_assert(OFF_HOP % 16 == 0 && OFF_BAR % 8 == 0 && OFF_K % 1024 == 0 && OFF_V % 1024 == 0,
                "shared-memory alignment");
  static_assert(SMEM <= 232448, "shared memory budget");
};

struct Params {
  const int32_t* q_pos;
  const int32_t* kv_pos;
  const int32_t* seg;  // packed sequences: segid per slot (q and kv), or NULL
  int BH, group, nseg, Lq_seg, Lk_seg, n_qtiles, causal;
  long long kv_valid;
  float scale_log2;
  void* o;
  int o_f32;
  float* lse;
  int* err;
  unsigned long long wait_ns;
};

template <bool SEG>  // SEG: packed sequences (segid array present)
__global__ void __launch_bounds__(kThreads, 1)
    fwd_wide_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using C = Cfg;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_q_full = bars;
  uint64_t* bar_k_full = bars + 1;             // [NSK]
  uint64_t* bar_k_empty = bar_k_full + C::NSK;  // [NSK]
  uint64_t* bar_v_full = bar_k_empty + C::NSK;
  uint64_t* bar_v_empty = bar_v_full + 1;
  uint64_t* bar_s_full = bar_v_empty + 1;
  uint64_t* bar_s_free = bar_s_full + 1;  // the softmax warps have read S_g
  uint64_t* bar_p_ready = bar_s_free + 1;
  uint64_t* bar_o_done = bar_p_ready + 1;  // PV_g completed (P buffer free, O current)
  uint64_t* bar_drain = bar_o_done + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  int4* s_hop = reinterpret_cast<int4*>(smem + C::OFF_HOP);
  float* s_xch = reinterpret_cast<float*>(smem + C::OFF_XCH);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // The 128-byte swizzle needs 1024-byte aligned tiles; otherwise nothing is
  // loaded or computed (every tile range is empty) and the error is recorded.
  const bool smem_ok = (smem_u32(smem) & 1023u) == 0;

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
    if (!smem_ok && p.err) atomicCAS(p.err, 0, SITE_FWD_LOAD);
    mbar_init(bar_q_full, 1);
    for (int i = 0; i < C::NSK; ++i) {
      mbar_init(&bar_k_full[i], 1);
      mbar_init(&bar_k_empty[i], 1);
    }
    mbar_init(bar_v_full, 1);
    mbar_init(bar_v_empty, 1);
    mbar_init(bar_s_full, 1);
    mbar_init(bar_s_free, 8);   // one arrival per softmax warp
    mbar_init(bar_p_ready, 8);
    mbar_init(bar_o_done, 1);
    mbar_init(bar_drain, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) tmem_alloc(s_tmem, C::T_COLS);

  // Per hop: visible 256-key tiles [first, n_vis) and unmasked ones [f_lo,
  // f_hi), partition points over the non-decreasing positions (and segids) of
  // the segment; one warp per hop.
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
  if (smem_ok)
    for (int t = 0; t < p.nseg; ++t) G += s_hop[t].y - s_hop[t].x;

  int issued_k = 0, issued_v = 0;  // producer bookkeeping for the drain

  if (warp >= 8) {
    regs_dec<kRegsLoad>();
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && G > 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      mbar_arrive_expect_tx(bar_q_full, C::QTILE);
      for (int b = 0; b < 2; ++b) tma_load_4d(sQ + b * C::QBOX, &tm_q, bar_q_full, b * 64, q0, r, bh);
      bool ok = true;
      // V_g is loaded after K_{g+1}: the key/tile coordinates of the last two
      // tiles are kept for that.
      int vs0 = 0, vj0 = 0, vs1 = 0, vj1 = 0;
      auto load_v = [&](int gv, int s, int j) -> bool {
        if (gv > 0 && !mbar_wait(bar_v_empty, (gv - 1) & 1, s_abort, p.wait_ns)) return false;
        mbar_arrive_expect_tx(bar_v_full, C::KTILE);
        for (int b = 0; b < 2; ++b) tma_load_4d(sV + b * C::KBOX, &tm_v, bar_v_full, b * 64, j * BN, s, kvh);
        ++issued_v;
        return true;
      };
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
          mbar_arrive_expect_tx(&bar_k_full[st], C::KTILE);
          for (int b = 0; b < 2; ++b)
            tma_load_4d(sK + st * C::KTILE + b * C::KBOX, &tm_k, &bar_k_full[st], b * 64, j * BN, s, kvh);
          ++issued_k;
          if (g >= 1 && !load_v(g - 1, (g & 1) ? vs0 : vs1, (g & 1) ? vj0 : vj1)) {
            ok = false;
            break;
          }
          if (g & 1) { vs1 = s; vj1 = j; } else { vs0 = s; vj0 = j; }
        }
      }
      if (ok && G > 0) ok = load_v(G - 1, ((G - 1) & 1) ? vs1 : vs0, ((G - 1) & 1) ? vj1 : vj0);
      if (!ok) record_failure(s_abort, p.err, SITE_FWD_LOAD);
    }
  } else if (warp == 9) {
    // ----------------------------------------------------------- MMA issue
    // The whole warp walks the schedule and waits; one elected lane issues.
    if (G > 0) {
      const uint32_t idesc_s = idesc_bf16_f32(BM, BN, 0, 0);
      const uint32_t idesc_o = idesc_bf16_f32(BM, D, 0, 1);
      const uint32_t sQa = smem_u32(sQ), sKa0 = smem_u32(sK), sVa = smem_u32(sV);
      bool ok = warp_wait(bar_q_full, 0, s_abort, p.wait_ns);
      // S_g = Q K_g^T: 128 x 256 into the score buffer
      auto issue_s = [&](int g) -> bool {
        const int st = g % C::NSK;
        if (!warp_wait(&bar_k_full[st], (g / C::NSK) & 1, s_abort, p.wait_ns)) return false;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ad = sdesc_sw128(sQa + (kk >> 2) * C::QBOX + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(sKa0 + st * C::KTILE + (kk >> 2) * C::KBOX + (kk & 3) * 32, 16, 1024);
            umma_ss(tmem, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar_s_full);
          umma_commit(&bar_k_empty[st]);
        }
        __syncwarp();
        return true;
      };
      // O += P_g V_g, P_g (bf16, 256 keys) from the P buffer, V_g MN-major
      auto issue_pv = [&](int g) -> bool {
        if (!warp_wait(bar_p_ready, g & 1, s_abort, p.wait_ns)) return false;
        if (!warp_wait(bar_v_full, g & 1, s_abort, p.wait_ns)) return false;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            umma_ts(tmem + C::T_O, tmem + C::T_P + kk * 8, sdesc_sw128(sVa + kk * 2048, C::KBOX, 1024), idesc_o,
                    (g > 0 || kk > 0) ? 1u : 0u);
          umma_commit(bar_o_done);
          umma_commit(bar_v_empty);
        }
        __syncwarp();
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int g = 0; g < G && ok; ++g) {
        if (g + 1 < G) {  // S_{g+1} as soon as the softmax warps hold S_g
          ok = warp_wait(bar_s_free, g & 1, s_abort, p.wait_ns) && issue_s(g + 1);
          if (!ok) break;
        }
        ok = issue_pv(g);
      }
      if (!ok && lane == 0) record_failure(s_abort, p.err, SITE_FWD_MMA);
    }
  }
  } else {
    regs_inc<kRegsSoftmax>();
    // -------------------------------------------------- softmax + epilogue
    const int quarter = warp & 3;
    const int half = warp >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const int meet = 1 + quarter;  // named barrier of the two warps of this quarter
    const bool row_valid = row < q_rows;
    const long long my_pos = row_valid ? qpos(p, r, q0 + row) : q_max;
    if (kDebugChecks && row_valid && q0 + row > 0) check_order(qpos(p, r, q0 + row - 1) <= my_pos, p.err, 6);
    const int my_seg = (SEG && row_valid) ? segat(p, r, q0 + row) : 1;  // odd: sees nothing
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    bool bad = false;  // a failed wait, reported at the next meeting
    int g = 0;
    for (int t = 0; t < p.nseg && ok; ++t) {
      const int s = ((r - t) % p.nseg + p.nseg) % p.nseg;
      const int nv = s_hop[t].y, f_lo = s_hop[t].z, f_hi = s_hop[t].w;
      for (int j = s_hop[t].x; j < nv; ++j, ++g) {
        // Visible keys of this row among this warp's 128: a run [klo, khi)
        // (all of them in an unmasked tile; a prefix without packed
        // sequences), found before the scores arrive by binary searches over
        // the keys' positions (and segids) held four per lane.
        int klo = 0, khi = 128;
        if (j < f_lo || j >= f_hi) {
          const int kh0 = j * BN + half * 128;
          const int n = max(0, min(128, p.Lk_seg - kh0));
          const long long kbase = static_cast<long long>(s) * p.Lk_seg + kh0;
          int kp4[4], ks4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int idx = 4 * lane + e;
            const bool inb = idx < n && in_bounds(kbase + idx, static_cast<long long>(p.nseg) * p.Lk_seg, p.err, 4);
            kp4[e] = inb ? (p.kv_pos ? __ldg(p.kv_pos + kbase + idx) : kh0 + idx) : INT_MAX;
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
        const bool got = !bad && warp_wait(bar_s_full, g & 1, s_abort, p.wait_ns);
        uint32_t sr[4][32];
        uint32_t pk[4][16];                           // P_g, bf16 pairs
        uint64_t sum4[4] = {0ull, 0ull, 0ull, 0ull};  // its eight partial row sums
        // P_g against the reference max m (0 while a row has none): exponent
        // arguments and row sums two keys at a time (f32x2).
        auto form_p = [&](float m) {
          const uint64_t sl2x2 = f32x2(sl2, sl2), nm2 = f32x2(-m, -m);
#pragma unroll
          for (int i = 0; i < 4; ++i) sum4[i] = 0ull;
#pragma unroll
          for (int h = 0; h < 4; ++h)  // 32 keys (16 packed columns) at a time
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float2 t = f32x2_split(
                  fma_f32x2(f32x2(__uint_as_float(sr[h][2 * i]), __uint_as_float(sr[h][2 * i + 1])), sl2x2, nm2));
              const float a = ex2_approx(t.x), b = ex2_approx(t.y);
              sum4[i & 3] = add_f32x2(sum4[i & 3], f32x2(a, b));
              pk[h][i] = pack_bf16x2(a, b);
            }
        };
        bool full = true;  // the full path: row max, exchange, lazy rescale
        if (got) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_base + half * 128 + c * 32, sr[c]);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_s_free);  // the next score product may overwrite S
          if (klo > 0 || khi < 128) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (c * 32 + i < klo || c * 32 + i >= khi) sr[c][i] = __float_as_uint(-INFINITY);
          }
          // Short path: P_g against the reference max kept so far, with no row
          // max. It stands unless a row of the quarter needs a new reference:
          // its first visible keys, or a half-row sum above 2^16 (some score
          // more than 9 above the reference, log2 units), where the full path
          // below takes over. Values below 2^16 keep the fp32 sums and the
          // bf16 P far from overflow; the result is exact either way.
          form_p(m_run == -INFINITY ? 0.f : m_run);
          const float2 s01 = f32x2_split(add_f32x2(sum4[0], sum4[1]));
          const float2 s23 = f32x2_split(add_f32x2(sum4[2], sum4[3]));
          const float lt = (s01.x + s01.y) + (s23.x + s23.y);
          full = (m_run == -INFINITY && klo < khi) || !(lt <= 65536.f);
        }
        bool pv_prev_done = g == 0;  // PV_{g-1}, the last reader of the P buffer, has completed
        // Both warps of the quarter meet here once per tile; any failed wait
        // also sends both into the full path, whose meeting reports it.
        if (bar_any(meet, 64, full)) {
          float pm = -INFINITY;
          if (got) {
            float mx8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mx8[i] = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
              for (int i = 0; i < 32; i += 2)
                mx8[(i >> 1) & 7] =
                    fmax3(mx8[(i >> 1) & 7], __uint_as_float(sr[c][i]), __uint_as_float(sr[c][i + 1]));
            pm = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
          }
          // Hand over the partial max; both warps leave together on any failure.
          s_xch[((g & 1) * 2 + half) * BM + row] = pm;
          if (bar_any(meet, 64, !got)) {
            record_failure(s_abort, p.err, SITE_FWD_SOFTMAX);
            ok = false;
            break;
          }
          // max is exact and commutative: both halves hold the same value
          float mx = fmaxf(pm, s_xch[((g & 1) * 2 + (half ^ 1)) * BM + row]);
          mx *= sl2;
          // Lazy rescale: keep the reference max unless the row max grew by > 8
          // (log2 units); exact either way.
          const bool need = mx > m_run + 8.f;
          float alpha = 1.f;
          const bool o_live = (g > 0) && (m_run != -INFINITY);
          if (need) {
            alpha = ex2_approx(m_run - mx);
            l_run *= alpha;
          }
          const bool warp_rescale = __any_sync(0xffffffffu, need && o_live) != 0;
          if (need) m_run = mx;
          // PV_{g-1} must be complete before O is rescaled.
          if (warp_rescale) {
            if (!warp_wait(bar_o_done, (g - 1) & 1, s_abort, p.wait_ns)) {
              record_failure(s_abort, p.err, SITE_FWD_SOFTMAX);
              bad = true;
              continue;
            }
            pv_prev_done = true;
            tc_fence_after();
            const uint32_t o_addr = tmem + lane_base + C::T_O + half * (D / 2);
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
              uint32_t orr[32];
              tmem_ld32(o_addr + c * 32, orr);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
              tmem_st32(o_addr + c * 32, orr);
            }
          }
          form_p(m_run == -INFINITY ? 0.f : m_run);
        }
        const uint32_t p_addr = tmem + lane_base + C::T_P + half * 64;
        if (!pv_prev_done) {
          if (!warp_wait(bar_o_done, (g - 1) & 1, s_abort, p.wait_ns)) {
            record_failure(s_abort, p.err, SITE_FWD_SOFTMAX);
            bad = true;
            continue;
          }
          tc_fence_after();
        }
#pragma unroll
        for (int h = 0; h < 4; ++h) tmem_st16(p_addr + h * 16, pk[h]);
        const float2 s01 = f32x2_split(add_f32x2(sum4[0], sum4[1])), s23 = f32x2_split(add_f32x2(sum4[2], sum4[3]));
        l_run += (s01.x + s01.y) + (s23.x + s23.y);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_p_ready);  // one arrival per warp
      }
    }

    // ---------------------------------------------------------- epilogue
    const long long out_row = (static_cast<long long>(bh) * p.nseg + r) * p.Lq_seg + q0 + row;
    const bool out_ok = !row_valid || in_bounds(out_row, static_cast<long long>(p.BH) * p.nseg * p.Lq_seg, p.err, 5);
    float l_tot = 0.f;
    if (ok && G > 0) {  // the two halves' row sums, added in a fixed order
      s_xch[((G & 1) * 2 + half) * BM + row] = l_run;
      if (bar_any(meet, 64, bad)) {
        record_failure(s_abort, p.err, SITE_FWD_EPILOGUE);
        ok = false;
      } else {
        l_tot = s_xch[((G & 1) * 2) * BM + row] + s_xch[((G & 1) * 2 + 1) * BM + row];
      }
    }
    const float inv_l = l_tot > 0.f ? 1.f / l_tot : 0.f;
    if (ok && G > 0) {
      if (!warp_wait(bar_o_done, (G - 1) & 1, s_abort, p.wait_ns)) {
        record_failure(s_abort, p.err, SITE_FWD_EPILOGUE);
        ok = false;
      }
    }
    if (ok) {
      if (G > 0) tc_fence_after();
      const uint32_t o_addr = tmem + lane_base + C::T_O + half * (D / 2);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t orr[32];
        if (G > 0) {
          tmem_ld32(o_addr + c * 32, orr);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) orr[i] = 0u;
        }
        if (row_valid && out_ok) {
          const long long col = half * (D / 2) + c * 32;
          if (p.o_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.o) + out_row * D + col);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(orr[4 * i]) * inv_l, __uint_as_float(orr[4 * i + 1]) * inv_l,
                                   __uint_as_float(orr[4 * i + 2]) * inv_l, __uint_as_float(orr[4 * i + 3]) * inv_l);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + out_row * D + col);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(orr[8 * i + 0]) * inv_l, __uint_as_float(orr[8 * i + 1]) * inv_l);
              w.y = pack_bf16x2(__uint_as_float(orr[8 * i + 2]) * inv_l, __uint_as_float(orr[8 * i + 3]) * inv_l);
              w.z = pack_bf16x2(__uint_as_float(orr[8 * i + 4]) * inv_l, __uint_as_float(orr[8 * i + 5]) * inv_l);
              w.w = pack_bf16x2(__uint_as_float(orr[8 * i + 6]) * inv_l, __uint_as_float(orr[8 * i + 7]) * inv_l);
              dst[i] = w;
            }
          }
        }
      }
      if (row_valid && out_ok && half == 0)
        p.lse[out_row] = l_tot > 0.f ? (m_run + __log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
    }
  }

  // ------------------------------------------------------------ teardown
  if (warp == 8 && lane == 0 && G > 0) {
    drain_wait(bar_q_full, 0);
    for (int g = max(0, issued_k - C::NSK); g < issued_k; ++g)
      drain_wait(&bar_k_full[g % C::NSK], (g / C::NSK) & 1);
    if (issued_v > 0) drain_wait(bar_v_full, (issued_v - 1) & 1);
  }
  if (warp == 9 && G > 0) {  // the lane that issued the products commits
    if (elect_one()) {
      umma_commit(bar_drain);
      if (!drain_wait(bar_drain, 0)) record_failure(s_abort, p.err, SITE_DRAIN);
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::T_COLS);
  }
}

}  // namespace

// One-tile forward over 256-key tiles (D = 128, bf16, at most 32 segments).
rattn_status launch_fwd_sm100_wide(const FwdArgs& a, const DevCtx& ctx) {
  using C = Cfg;
  if (a.D != D || a.dtype != RATTN_BF16 || a.nseg > kMaxHops) return RATTN_ERR_UNSUPPORTED;
  if (a.Lq_seg > INT32_MAX - BM || a.Lk_seg > INT32_MAX - BN) return RATTN_ERR_UNSUPPORTED;
  const int n_qtiles = static_cast<int>((a.Lq_seg + BM - 1) / BM);
  const long long grid = static_cast<long long>(a.BH) * a.nseg * n_qtiles;
  if (grid == 0) return RATTN_OK;
  if (grid > INT32_MAX) return RATTN_ERR_UNSUPPORTED;
  if (a.group < 1 || a.BH % a.group) return RATTN_ERR_INVALID_ARG;
  CUtensorMap tq, tk, tv;
  rattn_status st;
  if ((st = make_tmap_bf16(&tq, a.q, D, a.Lq_seg, a.nseg, a.BH, BM)) != RATTN_OK) return st;
  if ((st = make_tmap_bf16(&tk, a.k, D, a.Lk_seg, a.nseg, a.BH / a.group, BN)) != RATTN_OK) return st;
  if ((st = make_tmap_bf16(&tv, a.v, D, a.Lk_seg, a.nseg, a.BH / a.group, BN)) != RATTN_OK) return st;
  const void* kfn = a.seg ? reinterpret_cast<const void*>(&fwd_wide_kernel<true>)
                         : reinterpret_cast<const void*>(&fwd_wide_kernel<false>);
  if ((st = set_smem_attr(kfn, C::SMEM)) != RATTN_OK) return st;
  {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kfn) != cudaSuccess) return RATTN_ERR_CUDA;
    if (fa.numRegs != kLaunchRegs) return RATTN_ERR_UNSUPPORTED;  // the register split would not balance
  }
  Params p;
  p.q_pos = a.q_pos;
  p.kv_pos = a.kv_pos;
  p.seg = a.seg;
  p.BH = a.BH;
  p.group = a.group;
  p.nseg = a.nseg;
  p.Lq_seg = static_cast<int>(a.Lq_seg);
  p.Lk_seg = static_cast<int>(a.Lk_seg);
  p.n_qtiles = n_qtiles;
  p.causal = a.causal;
  p.kv_valid = a.kv_valid;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.o = a.o;
  p.o_f32 = a.o_f32;
  p.lse = a.lse;
  p.err = ctx.err_word;
  p.wait_ns = ctx.wait_ns;
  if (a.seg)
    fwd_wide_kernel<true><<<static_cast<unsigned>(grid), kThreads, C::SMEM, a.stream>>>(tq, tk, tv, p);
  else
    fwd_wide_kernel<false><<<static_cast<unsigned>(grid), kThreads, C::SMEM, a.stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? RATTN_OK : RATTN_ERR_CUDA;
}

}  // namespace rattn
