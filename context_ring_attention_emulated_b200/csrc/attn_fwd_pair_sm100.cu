// attn_fwd_pair_sm100.cu -- the ring / partial attention forward with two
// query tiles per CTA (sm_100a: tcgen05.mma, TMEM accumulators, TMA-staged
// K/V tiles). It computes exactly what attn_fwd_sm100.cu's kernel computes,
// in the same order per row, and gives bit-identical O and LSE; it differs in
// how the work is tiled, which suits long rows (see launch_fwd_sm100).
//
// What it computes ([CP-glossary] "How context parallelism works";
// [Ring-page] "Deep dive", "Technical insight"): every emulated rank keeps its
// query tiles fixed while the K/V blocks of the ring arrive hop by hop (rank r
// holds the block of rank (r - t) mod cp at hop t); each arriving block's
// scores are folded into a running row max and running normaliser, earlier
// partial sums being rescaled when the max grows, so the result equals full
// softmax attention. Tiles the causal position relation fully masks are
// skipped.
//
// One CTA owns two consecutive 128-row query tiles (Q0, Q1) of one (batch,
// head, rank); both attend every K/V tile of every hop in ring order, so each
// K/V tile staged in shared memory serves 256 query rows (half the K/V
// traffic per FLOP of the one-tile kernel). Warp roles (384 threads):
//   warp 0      TMA producer: Q0, Q1 once, then K (3 stages) and V (2
//               stages for D = 128) through rings of shared-memory buffers;
//   warp 1      TMEM allocation and tcgen05.mma issue (one elected lane of the warp), in
//               the order PV0(j), S0(j+1), PV1(j), S1(j+1): S_b = Q_b K^T
//               into tile b's score buffer, O_b += P_b V with P_b read from
//               TMEM; S_b(j+1) waits for PV_b(j), which reads P_b(j) there;
//   warps 2, 3  idle (they complete warpgroup 0, whose registers go to the
//               softmax warpgroups);
//   warps 4..7  softmax of Q0, warps 8..11 softmax of Q1, one thread per
//               query row (= TMEM lane), holding the whole 128-key score row
//               in registers: row max, lazy rescale of O_b (only when the max
//               grows by more than 2^8; O_b is idle then), exp2, row sum, P_b
//               packed to bf16 over its own scores; finally the epilogue.
// When a slice has an odd number of tiles, the last pair has no Q1: its
// MMAs are not issued and warps 8..11 idle.
// TMEM columns: S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D).
// Registers: launched at 168 a thread; warpgroup 0 shrinks to 56 and the
// softmax warpgroups grow to 224 (setmaxnreg); the host refuses to launch
// unless the kernel was built with exactly 168, so the split balances.
//
// Grouped key/value heads: query head h reads the K/V of head h / group.
// Packed sequences (the SEG instantiation): a key is visible only to queries
// carrying the same even segid.
#include <limits.h>
#include <math.h>

#include "debug_check.cuh"
#include "fwd_positions.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace rattn {
namespace {

constexpr int kThreads = 384;  // 12 warps
// Registers: launched at kLaunchRegs (12 warps, 3 per register-file
// partition); the producer/MMA warpgroup (warps 0..3, two of them idle)
// shrinks to kRegsLoad so that each softmax warpgroup can hold a whole
// 128-key score row per thread (kRegsSoftmax).
constexpr int kLaunchRegs = 168;
constexpr int kRegsLoad = 56;
constexpr int kRegsSoftmax = 224;
static_assert(kRegsLoad + 2 * kRegsSoftmax == 3 * kLaunchRegs, "register split must balance");
constexpr int BM = 128;  // query rows per tile (two tiles per CTA)
constexpr int BN = 128;  // keys per tile
constexpr int kMaxHops = 64;

template <int D>
struct Cfg {
  static constexpr int NSK = (D == 128) ? 3 : 4;  // K stages
  static constexpr int NSV = (D == 128) ? 2 : 4;  // V stages
  static constexpr int TILE = BM * D * 2;        // bytes of one 128 x D bf16 tile
  static constexpr int NBOX = D / 64;            // 64-element (128-byte) swizzle boxes per row
  static constexpr int BOX = BM * 128;           // bytes of one 128-row box
  static constexpr uint32_t T_O = 256;           // O0 at T_O, O1 at T_O + D
  static constexpr uint32_t T_COLS = 512;
  static constexpr int OFF_Q = 0;                // Q0, Q1
  static constexpr int OFF_K = OFF_Q + 2 * TILE;
  static constexpr int OFF_V = OFF_K + NSK * TILE;
  static constexpr int OFF_BAR = OFF_V + NSV * TILE;
  static constexpr int NBAR = 1 + 2 * NSK + 2 * NSV + 2 + 2 + 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_HOP = (OFF_MISC + 16 + 15) / 16 * 16;  // int4 tables: 16-byte aligned
  static constexpr int SMEM = OFF_HOP + 2 * kMaxHops * 16;
  static_assert(OFF_HOP % 16 == 0 && OFF_BAR % 8 == 0, "shared-memory alignment");
  static_assert(SMEM <= 232448, "shared memory budget");
};

struct Params {
  const int32_t* q_pos;
  const int32_t* kv_pos;
  const int32_t* seg;  // packed sequences: segid per slot (q and kv), or NULL
  int BH, group, nseg, Lq_seg, Lk_seg, n_qtiles, n_pairs, causal;
  long long kv_valid;
  float scale_log2;
  void* o;
  int o_f32;
  float* lse;
  int* err;
  unsigned long long wait_ns;
};

// Visible K/V tiles of one hop for a query range [qa, qb] (rows of rank r) and
// the sub-range with no masked element: x = first visible tile, y = end of
// the visible tiles, [z, w) = tiles fully visible to every row of the range.
// Keys are sorted by position (and by segid for packed sequences) within a
// segment, so every bound is the partition point of a predicate that holds on
// a prefix of a tile range; without packed sequences the visible tiles are a
// prefix. All 32 lanes of a warp call it together.
template <bool SEG>
__device__ int4 hop_ranges(const Params& p, int r, int s, int qa, int qb, int nk_tiles, int lane) {
  const long long q_min = qpos(p, r, qa), q_max = qpos(p, r, qb);
  const int sq_lo = SEG ? segat(p, r, qa) : 0;
  const int sq_hi = SEG ? segat(p, r, qb) : 0;
  const int first = SEG ? warp_partition_point(0, nk_tiles, lane, [&](int m) {
    return segat(p, s, min((m + 1) * BN, p.Lk_seg) - 1) < sq_lo;  // tile ends before the query segments
  }) : 0;
  const int n_vis = warp_partition_point(first, nk_tiles, lane, [&](int m) {
    const long long kmin = kpos(p, s, m * BN);
    return kmin < p.kv_valid && (!p.causal || kmin <= q_max) && (!SEG || segat(p, s, m * BN) <= sq_hi);
  });
  int f_lo = first, f_hi = first;
  const bool one_seg = !SEG || (sq_lo == sq_hi && (sq_lo & 1) == 0);
  if (one_seg && first < n_vis) {
    int a = first, b = n_vis;
    if (SEG) {  // tiles lying wholly in the query range's segment: [a, b)
      a = warp_partition_point(first, n_vis, lane, [&](int m) { return segat(p, s, m * BN) < sq_lo; });
      b = warp_partition_point(a, n_vis, lane, [&](int m) {
        return segat(p, s, min((m + 1) * BN, p.Lk_seg) - 1) <= sq_lo;
      });
    }
    f_lo = a;
    f_hi = warp_partition_point(a, b, lane, [&](int m) {  // leading tiles visible to every query row
      const bool complete = (m + 1) * BN <= p.Lk_seg;
      const long long kmax = kpos(p, s, min((m + 1) * BN, p.Lk_seg) - 1);
      return complete && kmax < p.kv_valid && (!p.causal || kmax <= q_min);
    });
  }
  return make_int4(first, n_vis, f_lo, f_hi);
}

template <int D, bool SEG>  // SEG: packed sequences (segid array present)
__global__ void __launch_bounds__(kThreads, 1)
    fwd_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using C = Cfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_q_full = bars;
  uint64_t* bar_k_full = bars + 1;
  uint64_t* bar_k_empty = bar_k_full + C::NSK;
  uint64_t* bar_v_full = bar_k_empty + C::NSK;
  uint64_t* bar_v_empty = bar_v_full + C::NSV;
  uint64_t* bar_s_full = bar_v_empty + C::NSV;  // [2]: S_b(j) in TMEM
  uint64_t* bar_p_ready = bar_s_full + 2;      // [2]: P_b(j) over it (one arrival per softmax warp)
  uint64_t* bar_o_done = bar_p_ready + 2;      // [2]: PV_b(j) completed
  uint64_t* bar_drain = bar_o_done + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  // per hop: the pair's visible tiles and tile 0's fully visible ones
  // (s_hop), tile 1's fully visible ones (s_hop1.z, .w)
  int4* s_hop = reinterpret_cast<int4*>(smem + C::OFF_HOP);
  int4* s_hop1 = s_hop + kMaxHops;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // The 128-byte swizzle needs 1024-byte aligned tiles; refuse to run otherwise.
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0 && p.err) atomicCAS(p.err, 0, SITE_FWD_LOAD);
    return;
  }

  // Work item: (batch, head) slowest, then rank, then tile pair, heaviest
  // first (largest local index, hence largest positions under every layout):
  // the CTAs resident at any time walk the same hop's K/V block together.
  int item = blockIdx.x;
  const int pq = p.n_pairs - 1 - (item % p.n_pairs);
  item /= p.n_pairs;
  const int r = item % p.nseg;
  const int bh = item / p.nseg;
  const int kvh = bh / p.group;  // (batch, key/value head): query heads of a group are contiguous
  const int qa0 = pq * 2 * BM;                             // first row of Q0
  const int rows0 = min(BM, p.Lq_seg - qa0);
  const int rows1 = max(0, min(BM, p.Lq_seg - qa0 - BM));  // Q1 may be empty (odd tile count)
  const int q_last = qa0 + rows0 + rows1 - 1;              // last valid row of the pair
  const bool two = rows1 > 0;                              // Q1 holds rows: S1 / PV1 are issued
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
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar_s_full[b], 1);
      mbar_init(&bar_p_ready[b], 4);  // one arrival per softmax warp of the tile
      mbar_init(&bar_o_done[b], 1);
    }
    mbar_init(bar_drain, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(s_tmem, C::T_COLS);

  for (int t = warp; t < p.nseg; t += kThreads / 32) {  // one warp per hop
    const int s = ((r - t) % p.nseg + p.nseg) % p.nseg;
    const int4 all = hop_ranges<SEG>(p, r, s, qa0, q_last, nk_tiles, lane);
    const int4 h0 = hop_ranges<SEG>(p, r, s, qa0, qa0 + rows0 - 1, nk_tiles, lane);
    const int4 h1 = rows1 > 0 ? hop_ranges<SEG>(p, r, s, qa0 + BM, q_last, nk_tiles, lane) : make_int4(0, 0, 0, 0);
    if (lane == 0) {
      s_hop[t] = make_int4(all.x, all.y, h0.z, h0.w);
      s_hop1[t] = h1;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  int G = 0;
  for (int t = 0; t < p.nseg; ++t) G += s_hop[t].y - s_hop[t].x;

  int issued_k = 0, issued_v = 0;  // producer bookkeeping for the drain

  if (warp < 4) {
    regs_dec<kRegsLoad>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && G > 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      mbar_arrive_expect_tx(bar_q_full, 2 * C::TILE);
      for (int b = 0; b < 2; ++b)
        for (int x = 0; x < C::NBOX; ++x)
          tma_load_4d(sQ + b * C::TILE + x * C::BOX, &tm_q, bar_q_full, x * 64, qa0 + b * BM, r, bh);
      bool ok = true;
      int g = 0;
      for (int t = 0; t < p.nseg && ok; ++t) {
        const int s = ((r - t) % p.nseg + p.nseg) % p.nseg;
        const int nv = s_hop[t].y;
        for (int j = s_hop[t].x; j < nv; ++j, ++g) {
          const int st = g % C::NSK;
          const uint32_t u = g / C::NSK;
          if (u > 0 && !mbar_wait(&bar_k_empty[st], (u - 1) & 1, s_abort, p.wait_ns)) {
            record_failure(s_abort, p.err, SITE_FWD_LOAD);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_k_full[st], C::TILE);
          for (int x = 0; x < C::NBOX; ++x)
            tma_load_4d(sK + st * C::TILE + x * C::BOX, &tm_k, &bar_k_full[st], x * 64, j * BN, s, kvh);
          ++issued_k;
          const int sv = g % C::NSV;
          const uint32_t uv = g / C::NSV;
          if (uv > 0 && !mbar_wait(&bar_v_empty[sv], (uv - 1) & 1, s_abort, p.wait_ns)) {
            record_failure(s_abort, p.err, SITE_FWD_LOAD);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_v_full[sv], C::TILE);
          for (int x = 0; x < C::NBOX; ++x)
            tma_load_4d(sV + sv * C::TILE + x * C::BOX, &tm_v, &bar_v_full[sv], x * 64, j * BN, s, kvh);
          ++issued_v;
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issue
    if (G > 0) {  // the whole warp walks the schedule and waits; one elected lane issues
      const uint32_t idesc_s = idesc_bf16_f32(BM, BN, 0, 0);
      const uint32_t idesc_o = idesc_bf16_f32(BM, D, 0, 1);
      auto wt = [&](uint64_t* bar, uint32_t parity) { return warp_wait(bar, parity, s_abort, p.wait_ns); };
      // S_b(g) = Q_b K_g^T into tile b's score buffer; S_b(g) overwrites
      // P_b(g-1), so it waits for PV_b(g-1) to complete.
      auto issue_s = [&](int b, int g) -> bool {
        const int st = g % C::NSK;
        if (b == 0 && !wt(&bar_k_full[st], (g / C::NSK) & 1)) return false;
        if (g > 0 && !wt(&bar_o_done[b], (g - 1) & 1)) return false;
        tc_fence_after();
        if (elect_one()) {
          const uint32_t sQa = smem_u32(sQ + b * C::TILE);
          const uint32_t sKa = smem_u32(sK + st * C::TILE);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
            umma_ss(tmem + b * 128, sdesc_sw128(sQa + off, 16, 1024), sdesc_sw128(sKa + off, 16, 1024), idesc_s,
                    kk > 0 ? 1u : 0u);
          }
          umma_commit(&bar_s_full[b]);
          if (b == (two ? 1 : 0)) umma_commit(&bar_k_empty[st]);  // S0(g), S1(g) were K_g's readers
        }
        __syncwarp();
        return true;
      };
      // O_b += P_b(g) V_g with P_b read from the first 64 columns of its buffer
      auto issue_pv = [&](int b, int g) -> bool {
        const int st = g % C::NSV;
        if (!wt(&bar_p_ready[b], g & 1)) return false;
        if (b == 0 && !wt(&bar_v_full[st], (g / C::NSV) & 1)) return false;
        tc_fence_after();
        if (elect_one()) {
          const uint32_t sVa = smem_u32(sV + st * C::TILE);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            // V tile as an MN-major B operand: 16 keys = two 8-row swizzle atoms.
            const uint64_t bd = sdesc_sw128(sVa + kk * 2048, C::BOX, 1024);
            umma_ts(tmem + C::T_O + b * D, tmem + b * 128 + kk * 8, bd, idesc_o, (g > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bar_o_done[b]);
          if (b == (two ? 1 : 0)) umma_commit(&bar_v_empty[st]);  // PV0(g), PV1(g) were V_g's readers
        }
        __syncwarp();
        return true;
      };
      bool ok = warp_wait(bar_q_full, 0, s_abort, p.wait_ns);
      ok = ok && issue_s(0, 0) && (!two || issue_s(1, 0));
      for (int g = 0; g < G && ok; ++g) {
        ok = issue_pv(0, g);
        if (ok && g + 1 < G) ok = issue_s(0, g + 1);
        if (two) {
          if (ok) ok = issue_pv(1, g);
          if (ok && g + 1 < G) ok = issue_s(1, g + 1);
        }
      }
      if (!ok && lane == 0) record_failure(s_abort, p.err, SITE_FWD_MMA);
    }
  }
  } else if (warp >= 8 && !two) {
    regs_inc<kRegsSoftmax>();  // Q1 is empty: this warpgroup has nothing to do
  } else {
    regs_inc<kRegsSoftmax>();
    // -------------------------------------------------- softmax + epilogue
    const int b = (warp - 4) >> 2;  // query tile of this warpgroup
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const int q0 = qa0 + b * BM;
    const int q_rows = b == 0 ? rows0 : rows1;
    const bool row_valid = row < q_rows;
    const long long my_pos = row_valid ? qpos(p, r, q0 + row) : qpos(p, r, q_last);
    if (kDebugChecks && row_valid && q0 + row > 0) check_order(qpos(p, r, q0 + row - 1) <= my_pos, p.err, 6);
    const int my_seg = (SEG && row_valid) ? segat(p, r, q0 + row) : 1;  // odd: sees nothing
    const float sl2 = p.scale_log2;
    const int4* hop_b = b == 0 ? s_hop : s_hop1;
    const uint32_t s_addr = tmem + lane_base + b * 128;
    const uint32_t o_addr = tmem + lane_base + C::T_O + b * D;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    int g = 0;
    for (int t = 0; t < p.nseg && ok; ++t) {
      const int s = ((r - t) % p.nseg + p.nseg) % p.nseg;
      const int nv = s_hop[t].y, f_lo = hop_b[t].z, f_hi = hop_b[t].w;
      for (int j = s_hop[t].x; j < nv; ++j, ++g) {
        if (!warp_wait(&bar_s_full[b], g & 1, s_abort, p.wait_ns)) {
          record_failure(s_abort, p.err, SITE_FWD_SOFTMAX);
          ok = false;
          break;
        }
        tc_fence_after();
        // Visible keys of this row in the tile: [klo, khi) (all of them in a
        // tile with no masked element). In a masked tile the keys' positions
        // and segids are spread over the warp (four per lane, coalesced
        // loads) and every row's bounds come from binary searches over them
        // through shuffles (eight steps cover 128 keys; all lanes take every
        // step). Without packed sequences the run is a prefix.
        int klo = 0, khi = BN;
        const bool masked = j < f_lo || j >= f_hi;
        if (masked) {
          const int n = min(BN, p.Lk_seg - j * BN);
          const long long kbase = static_cast<long long>(s) * p.Lk_seg + j * BN;
          int kp4[4], ks4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int idx = 4 * lane + e;
            const bool inb = idx < n && in_bounds(kbase + idx, static_cast<long long>(p.nseg) * p.Lk_seg, p.err, 4);
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
        auto mask_chunk = [&](uint32_t (&v)[32], int c0) {
          if (masked) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c0 + i < klo || c0 + i >= khi) v[i] = __float_as_uint(-INFINITY);
          }
        };
        auto chunk_max = [&](float (&mx8)[8], const uint32_t (&v)[32]) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            mx8[(i >> 2) & 7] = fmax3(mx8[(i >> 2) & 7], fmax3(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                                                              __uint_as_float(v[i + 2])),
                                      __uint_as_float(v[i + 3]));
        };
        // The row max over the whole row, held in registers.
        uint32_t sa[32], sb[32], sc[32], sd[32];
        tmem_ld32(s_addr, sa);
        tmem_ld32(s_addr + 32, sb);
        tmem_ld32(s_addr + 64, sc);
        tmem_ld32(s_addr + 96, sd);
        tmem_wait_ld();
        mask_chunk(sa, 0);
        mask_chunk(sb, 32);
        mask_chunk(sc, 64);
        mask_chunk(sd, 96);
        float mx8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = -INFINITY;
        chunk_max(mx8, sa);
        chunk_max(mx8, sb);
        chunk_max(mx8, sc);
        chunk_max(mx8, sd);
        float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                         fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        mx *= sl2;
        // Lazy rescale: keep the reference max unless the row max grew by > 8
        // (log2 units), so exp2 values stay <= 256; exact either way. O_b is
        // idle here: PV_b(g-1) completed before S_b(g) was issued, and
        // PV_b(g) waits for this warpgroup's P.
        const bool need = mx > m_run + 8.f;
        float alpha = 1.f;
        const bool o_live = (g > 0) && (m_run != -INFINITY);
        if (need) {
          alpha = ex2_approx(m_run - mx);
          l_run *= alpha;
        }
        const bool warp_rescale = __any_sync(0xffffffffu, need && o_live) != 0;
        if (need) m_run = mx;
        if (warp_rescale) {
#pragma unroll 1
          for (int c = 0; c < D / 16; ++c) {
            uint32_t orr[16];
            tmem_ld16(o_addr + c * 16, orr);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
            tmem_st16(o_addr + c * 16, orr);
          }
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        float sum8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) sum8[i] = 0.f;
        // P = exp2(S scale log2e - m) for one 32-key chunk, packed to bf16
        // into 16 columns of its own buffer.
        auto exp_chunk = [&](const uint32_t (&v)[32], int c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float xa = fmaf(__uint_as_float(v[2 * i]), sl2, -m_use);
            const float xb = fmaf(__uint_as_float(v[2 * i + 1]), sl2, -m_use);
            const float ea = ex2_approx(xa);
            const float eb = ex2_approx(xb);
            sum8[i & 7] += ea + eb;
            pk[i] = pack_bf16x2(ea, eb);
          }
          tmem_st16(s_addr + c * 16, pk);
        };
        exp_chunk(sa, 0);
        exp_chunk(sb, 1);
        exp_chunk(sc, 2);
        exp_chunk(sd, 3);
        l_run += ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_p_ready[b]);  // one arrival per warp
      }
    }

    // ---------------------------------------------------------- epilogue
    // A row with no visible key has m_run = -inf: O = 0, LSE = -inf.
    const long long out_row = (static_cast<long long>(bh) * p.nseg + r) * p.Lq_seg + q0 + row;
    const bool out_ok = !row_valid || in_bounds(out_row, static_cast<long long>(p.BH) * p.nseg * p.Lq_seg, p.err, 5);
    const bool seen = m_run != -INFINITY && l_run > 0.f;
    const float inv_l = seen ? 1.f / l_run : 0.f;
    if (ok && G > 0) {
      if (!warp_wait(&bar_o_done[b], (G - 1) & 1, s_abort, p.wait_ns)) {
        record_failure(s_abort, p.err, SITE_FWD_EPILOGUE);
        ok = false;
      }
    }
    if (ok) {
      if (G > 0) tc_fence_after();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t orr[32];
        if (G > 0) {
          tmem_ld32(o_addr + c * 32, orr);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) orr[i] = 0u;
        }
        if (row_valid && out_ok) {
          if (p.o_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.o) + out_row * D + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(orr[4 * i]) * inv_l, __uint_as_float(orr[4 * i + 1]) * inv_l,
                                   __uint_as_float(orr[4 * i + 2]) * inv_l, __uint_as_float(orr[4 * i + 3]) * inv_l);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + out_row * D + c * 32);
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
      if (row_valid && out_ok) p.lse[out_row] = seen ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
    }
  }

  // ------------------------------------------------------------ teardown
  // Nothing may still write shared memory or TMEM when the CTA retires:
  // the producer waits for every copy it issued, the MMA thread for every
  // MMA it issued (both with a fixed limit, independent of the test hook).
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
rattn_status launch(const FwdArgs& a, const DevCtx& ctx) {
  using C = Cfg<D>;
  if (a.Lq_seg > INT32_MAX - 2 * BM || a.Lk_seg > INT32_MAX - BN) return RATTN_ERR_UNSUPPORTED;
  if (a.nseg > kMaxHops) return RATTN_ERR_UNSUPPORTED;
  const int n_qtiles = static_cast<int>((a.Lq_seg + BM - 1) / BM);
  const int n_pairs = (n_qtiles + 1) / 2;
  const long long grid = static_cast<long long>(a.BH) * a.nseg * n_pairs;
  if (grid == 0) return RATTN_OK;
  if (grid > INT32_MAX) return RATTN_ERR_UNSUPPORTED;
  CUtensorMap tq, tk, tv;
  rattn_status st;
  if ((st = make_tmap_bf16(&tq, a.q, D, a.Lq_seg, a.nseg, a.BH, BM)) != RATTN_OK) return st;
  if (a.group < 1 || a.BH % a.group) return RATTN_ERR_INVALID_ARG;
  if ((st = make_tmap_bf16(&tk, a.k, D, a.Lk_seg, a.nseg, a.BH / a.group, BN)) != RATTN_OK) return st;
  if ((st = make_tmap_bf16(&tv, a.v, D, a.Lk_seg, a.nseg, a.BH / a.group, BN)) != RATTN_OK) return st;
  const void* kfn = a.seg ? reinterpret_cast<const void*>(&fwd_pair_kernel<D, true>)
                         : reinterpret_cast<const void*>(&fwd_pair_kernel<D, false>);
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
  p.n_pairs = n_pairs;
  p.causal = a.causal;
  p.kv_valid = a.kv_valid;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.o = a.o;
  p.o_f32 = a.o_f32;
  p.lse = a.lse;
  p.err = ctx.err_word;
  p.wait_ns = ctx.wait_ns;
  if (a.seg)
    fwd_pair_kernel<D, true><<<static_cast<unsigned>(grid), kThreads, C::SMEM, a.stream>>>(tq, tk, tv, p);
  else
    fwd_pair_kernel<D, false><<<static_cast<unsigned>(grid), kThreads, C::SMEM, a.stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? RATTN_OK : RATTN_ERR_CUDA;
}

}  // namespace

rattn_status launch_fwd_sm100_pair(const FwdArgs& a, const DevCtx& ctx) {
  if (a.D == 128) return launch<128>(a, ctx);
  if (a.D == 64) return launch<64>(a, ctx);
  return RATTN_ERR_UNSUPPORTED;
}

}  // namespace rattn
