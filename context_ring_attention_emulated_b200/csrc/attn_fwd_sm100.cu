// attn_fwd_sm100.cu -- ring / partial attention forward on the sm_100a tensor
// cores (tcgen05.mma, TMEM accumulators, TMA-staged K/V tiles).
//
// What it computes ([CP-glossary] "How context parallelism works";
// [Ring-page] "Deep dive", "Technical insight"): every emulated rank keeps its
// query tile fixed while the K/V blocks of the ring arrive hop by hop (rank r
// holds the block of rank (r - t) mod cp at hop t); each arriving block's
// scores are folded into a running row max and running normaliser, earlier
// partial sums being rescaled when the max grows, so the result equals full
// softmax attention. Tiles that the causal position relation fully masks are
// skipped ([Megatron-CP] "Symmetric chunk assignment": the point of causal
// kernels skipping the upper triangle).
//
// One CTA owns one 128-row query tile of one (batch, head, rank) and walks
// every K/V tile of every hop in ring order. Warp roles:
//   warp 0      TMA producer: Q once, then K and V tiles through a
//               NS-stage ring of shared-memory buffers (the emulated KV hop:
//               the next block's loads run while the current block's MMAs do);
//   warp 1      allocates TMEM and issues tcgen05.mma from one elected lane:
//               S_g = Q K_g^T into one of three TMEM score buffers, running
//               three tiles ahead of O += P_g V_g (P read from TMEM), so the
//               score MMAs never wait on the previous tile's softmax;
//   warps 2..5  softmax, one thread per query row (= TMEM lane): row max,
//               lazy rescale of O (only when the max grows by more than
//               2^8), exp2, row sum, P packed to bf16 into TMEM; finally the
//               epilogue O / l and LSE.
// TMEM columns: S0 [0,128) S1 [128,256) S2 [256,384) O [384,384+D); P_g is
// written over the first 64 columns of its own score buffer. The MMA that
// next overwrites that buffer (S_{g+3}) is issued only after the PV MMA
// reading P_g has completed.
//
// Grouped key/value heads: query head h reads the K/V of head h / group.
// Packed sequences (the SEG instantiation; ring calls use the other one): a
// key is visible only to queries carrying the same even segid, so the visible
// tiles of a hop form a range rather than a prefix, and masked rows keep a
// contiguous run of keys.
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
  static constexpr int NS = (D == 128) ? 3 : 4;
  static constexpr int TILE = BM * D * 2;  // bytes of one 128 x D bf16 tile
  static constexpr int NBOX = D / 64;      // 64-element (128-byte) swizzle boxes per row
  static constexpr int BOX = BM * 128;     // bytes of one 128-row box
  static constexpr int NSB = 3;  // TMEM score buffers; P_g is written over its own scores
  static constexpr uint32_t T_O = 128 * NSB;
  static constexpr uint32_t T_COLS = 512;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + TILE;
  static constexpr int OFF_V = OFF_K + NS * TILE;
  static constexpr int OFF_BAR = OFF_V + NS * TILE;
  static constexpr int NBAR = 1 + 4 * NS + NSB + NSB + NSB + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_HOP = (OFF_MISC + 16 + 15) / 16 * 16;  // int4 table: 16-byte aligned
  static constexpr int SMEM = OFF_HOP + kMaxHops * 16 + 1024;        // + alignment slack
  static_assert(OFF_HOP % 16 == 0 && OFF_BAR % 8 == 0, "shared-memory alignment");
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

template <int D, bool SEG>  // SEG: packed sequences (segid array present)
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_q_full = bars;
  uint64_t* bar_k_full = bars + 1;
  uint64_t* bar_k_empty = bar_k_full + C::NS;
  uint64_t* bar_v_full = bar_k_empty + C::NS;
  uint64_t* bar_v_empty = bar_v_full + C::NS;
  uint64_t* bar_s_full = bar_v_empty + C::NS;     // [NSB]
  uint64_t* bar_p_ready = bar_s_full + C::NSB;    // [NSB]
  // o_done[b]: PV_g with g % NSB == b completed. A parity wait is only sound
  // when the waiter knows the previous phase completed; with one barrier per
  // score buffer that previous phase is PV_{g-NSB}, which every waiter has
  // already observed (its S_g was issued after it).
  uint64_t* bar_o_done = bar_p_ready + C::NSB;  // [NSB]
  uint64_t* bar_drain = bar_o_done + C::NSB;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  // per hop: x = first visible K/V tile, y = end of the visible tiles,
  // [z, w) = tiles with no masked element
  int4* s_hop = reinterpret_cast<int4*>(smem + C::OFF_HOP);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work item: (batch, head) slowest, then rank, then query tile, heaviest
  // first (largest local index, hence largest positions under every layout).
  // The CTAs resident at any time then belong to one rank of one head and
  // walk the same hop's K/V block at about the same time, so the block is
  // read from HBM about once per wave even when a head's K/V exceed L2.
  int item = blockIdx.x;
  const int qt = p.n_qtiles - 1 - (item % p.n_qtiles);
  item /= p.n_qtiles;
  const int r = item % p.nseg;
  const int bh = item / p.nseg;
  const int kvh = bh / p.group;  // (batch, key/value head): query heads of a group are contiguous
  const int q0 = qt * BM;
  const int q_rows = min(BM, p.Lq_seg - q0);
  const long long q_min = qpos(p, r, q0);
  const long long q_max = qpos(p, r, q0 + q_rows - 1);
  const int nk_tiles = (p.Lk_seg + BN - 1) / BN;

  if (threadIdx.x == 0) {
    mbar_init(bar_q_full, 1);
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(&bar_k_full[i], 1);
      mbar_init(&bar_k_empty[i], 1);
      mbar_init(&bar_v_full[i], 1);
      mbar_init(&bar_v_empty[i], 1);
    }
    for (int i = 0; i < C::NSB; ++i) {
      mbar_init(&bar_s_full[i], 1);
      mbar_init(&bar_p_ready[i], 4);  // one arrival per softmax warp
    }
    for (int i = 0; i < C::NSB; ++i) mbar_init(&bar_o_done[i], 1);
    mbar_init(bar_drain, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(s_tmem, C::T_COLS);

  // Per hop: the K/V tiles not fully masked form a range [first, n_vis) and
  // the tiles with no masked element a range [f_lo, f_hi) inside it; keys are
  // sorted by position (and by segid for packed sequences) within a segment,
  // so every bound is the partition point of a predicate that holds on a
  // prefix of a tile range. Without packed sequences the visible tiles are a
  // prefix. One warp per hop, 32-way searches (two rounds of loads for up to
  // 1024 tiles).
  for (int t = warp; t < p.nseg; t += kThreads / 32) {
    const int s = ((r - t) % p.nseg + p.nseg) % p.nseg;
    const int sq_lo = SEG ? segat(p, r, q0) : 0;
    const int sq_hi = SEG ? segat(p, r, q0 + q_rows - 1) : 0;
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
      if (SEG) {  // tiles lying wholly in the query tile's segment: [a, b)
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
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      mbar_arrive_expect_tx(bar_q_full, C::TILE);
      for (int b = 0; b < C::NBOX; ++b) tma_load_4d(sQ + b * C::BOX, &tm_q, bar_q_full, b * 64, q0, r, bh);
      bool ok = true;
      int g = 0;
      for (int t = 0; t < p.nseg && ok; ++t) {
        const int s = ((r - t) % p.nseg + p.nseg) % p.nseg;
        const int nv = s_hop[t].y;
        for (int j = s_hop[t].x; j < nv; ++j, ++g) {
          const int st = g % C::NS;
          const uint32_t u = g / C::NS;
          if (u > 0 && !mbar_wait(&bar_k_empty[st], (u - 1) & 1, s_abort, p.wait_ns)) {
            record_failure(s_abort, p.err, SITE_FWD_LOAD);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_k_full[st], C::TILE);
          for (int b = 0; b < C::NBOX; ++b)
            tma_load_4d(sK + st * C::TILE + b * C::BOX, &tm_k, &bar_k_full[st], b * 64, j * BN, s, kvh);
          ++issued_k;
          if (u > 0 && !mbar_wait(&bar_v_empty[st], (u - 1) & 1, s_abort, p.wait_ns)) {
            record_failure(s_abort, p.err, SITE_FWD_LOAD);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_v_full[st], C::TILE);
          for (int b = 0; b < C::NBOX; ++b)
            tma_load_4d(sV + st * C::TILE + b * C::BOX, &tm_v, &bar_v_full[st], b * 64, j * BN, s, kvh);
          ++issued_v;
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issue
    if (G > 0) {  // the whole warp walks the schedule and waits; one elected lane issues
      const uint32_t idesc_s = idesc_bf16_f32(BM, BN, 0, 0);
      const uint32_t idesc_o = idesc_bf16_f32(BM, D, 0, 1);
      const uint32_t sQa = smem_u32(sQ);
      bool ok = warp_wait(bar_q_full, 0, s_abort, p.wait_ns);
      // S_g = Q K_g^T into score buffer g % NSB
      auto issue_s = [&](int g) -> bool {
        const int st = g % C::NS;
        if (!warp_wait(&bar_k_full[st], (g / C::NS) & 1, s_abort, p.wait_ns)) return false;
        tc_fence_after();
        if (elect_one()) {
          const uint32_t d_s = tmem + (g % C::NSB) * 128;
          const uint32_t sKa = smem_u32(sK + st * C::TILE);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
            const uint64_t ad = sdesc_sw128(sQa + off, 16, 1024);
            const uint64_t bd = sdesc_sw128(sKa + off, 16, 1024);
            umma_ss(d_s, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
          }
          umma_commit(&bar_s_full[g % C::NSB]);
          umma_commit(&bar_k_empty[st]);
        }
        __syncwarp();
        return true;
      };
      // O += P_j V_j with P_j read from the first 64 columns of its score buffer
      auto issue_pv = [&](int j) -> bool {
        if (!warp_wait(&bar_p_ready[j % C::NSB], (j / C::NSB) & 1, s_abort, p.wait_ns)) return false;
        const int st = j % C::NS;
        if (!warp_wait(&bar_v_full[st], (j / C::NS) & 1, s_abort, p.wait_ns)) return false;
        tc_fence_after();
        if (elect_one()) {
          const uint32_t a_t = tmem + (j % C::NSB) * 128;
          const uint32_t sVa = smem_u32(sV + st * C::TILE);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            // V tile as an MN-major B operand: 16 keys = two 8-row swizzle atoms.
            const uint64_t bd = sdesc_sw128(sVa + kk * 2048, C::BOX, 1024);
            umma_ts(tmem + C::T_O, a_t + kk * 8, bd, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bar_o_done[j % C::NSB]);
          umma_commit(&bar_v_empty[st]);
        }
        __syncwarp();
        return true;
      };

      // S runs NSB tiles ahead of PV: S_0..S_{NSB-1}, then PV_g, S_{g+NSB}, ...
      // S_{g+NSB} overwrites P_g's buffer, so it is issued only once PV_g has
      // completed (issue order alone does not keep a later MMA's accumulator
      // writes behind an earlier MMA's TMEM operand reads).
      for (int g = 0; g < min(G, C::NSB) && ok; ++g) ok = issue_s(g);
      for (int g = 0; g < G && ok; ++g) {
        ok = issue_pv(g);
        if (ok && g + C::NSB < G) {
          ok = warp_wait(&bar_o_done[g % C::NSB], (g / C::NSB) & 1, s_abort, p.wait_ns);
          if (ok) ok = issue_s(g + C::NSB);
        }
      }
      if (!ok && lane == 0) record_failure(s_abort, p.err, SITE_FWD_MMA);
    }
  } else {
    // -------------------------------------------------- softmax + epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const bool row_valid = row < q_rows;
    const long long my_pos = row_valid ? qpos(p, r, q0 + row) : q_max;
    if (kDebugChecks && row_valid && q0 + row > 0) check_order(qpos(p, r, q0 + row - 1) <= my_pos, p.err, 6);
    const int my_seg = (SEG && row_valid) ? segat(p, r, q0 + row) : 1;  // odd: sees nothing
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    int g = 0;
    for (int t = 0; t < p.nseg && ok; ++t) {
      const int s = ((r - t) % p.nseg + p.nseg) % p.nseg;
      const int nv = s_hop[t].y, f_lo = s_hop[t].z, f_hi = s_hop[t].w;
      for (int j = s_hop[t].x; j < nv; ++j, ++g) {
        if (!warp_wait(&bar_s_full[g % C::NSB], (g / C::NSB) & 1, s_abort, p.wait_ns)) {
          record_failure(s_abort, p.err, SITE_FWD_SOFTMAX);
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sr[4][32];
        const uint32_t s_addr = tmem + lane_base + (g % C::NSB) * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + c * 32, sr[c]);
        tmem_wait_ld();
        if (j < f_lo || j >= f_hi) {
          // Masked tile: the visible keys of this row form a contiguous run
          // [klo, khi) of the tile (a prefix without packed sequences). The
          // tile's key positions and segids are spread over the warp (four
          // per lane, coalesced loads) and every row's bounds come from
          // binary searches over them through shuffles (eight steps cover 128
          // keys; all lanes take every step).
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
          int klo = 0;
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
          const int khi = lo;
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c * 32 + i < klo || c * 32 + i >= khi) sr[c][i] = __float_as_uint(-INFINITY);
        }
        float mx8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; i += 2)
            mx8[(i >> 1) & 7] =
                fmax3(mx8[(i >> 1) & 7], __uint_as_float(sr[c][i]), __uint_as_float(sr[c][i + 1]));
        float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                         fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        mx *= sl2;
        // Lazy rescale: keep the reference max unless the row max grew by > 8
        // (log2 units), so exp2 values stay <= 256; exact either way.
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
          if (!warp_wait(&bar_o_done[(g - 1) % C::NSB], ((g - 1) / C::NSB) & 1, s_abort, p.wait_ns)) {
            record_failure(s_abort, p.err, SITE_FWD_SOFTMAX);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t o_addr = tmem + lane_base + C::T_O;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t orr[32];
            tmem_ld32(o_addr + c * 32, orr);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
            tmem_st32(o_addr + c * 32, orr);
          }
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        float sum8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) sum8[i] = 0.f;
        const uint32_t p_addr = s_addr;  // P over the scores, all already in registers
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int c0 = h * 64 + 2 * i;
            const float a = ex2_approx(fmaf(__uint_as_float(sr[c0 >> 5][c0 & 31]), sl2, -m_use));
            const float b = ex2_approx(fmaf(__uint_as_float(sr[(c0 + 1) >> 5][(c0 + 1) & 31]), sl2, -m_use));
            sum8[i & 7] += a + b;
            pk[i] = pack_bf16x2(a, b);
          }
          tmem_st32(p_addr + h * 32, pk);
        }
        l_run += ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_p_ready[g % C::NSB]);  // one arrival per warp
      }
    }

    // ---------------------------------------------------------- epilogue
    const long long out_row = (static_cast<long long>(bh) * p.nseg + r) * p.Lq_seg + q0 + row;
    const bool out_ok = !row_valid || in_bounds(out_row, static_cast<long long>(p.BH) * p.nseg * p.Lq_seg, p.err, 5);
    const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
    if (ok && G > 0) {
      if (!warp_wait(&bar_o_done[(G - 1) % C::NSB], ((G - 1) / C::NSB) & 1, s_abort, p.wait_ns)) {
        record_failure(s_abort, p.err, SITE_FWD_EPILOGUE);
        ok = false;
      }
    }
    if (ok) {
      if (G > 0) tc_fence_after();
      const uint32_t o_addr = tmem + lane_base + C::T_O;
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
      if (row_valid && out_ok)
        p.lse[out_row] = l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
    }
  }

  // ------------------------------------------------------------ teardown
  // Nothing may still write shared memory or TMEM when the CTA retires:
  // the producer waits for every copy it issued, the MMA thread for every
  // MMA it issued (both with a fixed limit, independent of the test hook).
  if (warp == 0 && lane == 0 && G > 0) {
    drain_wait(bar_q_full, 0);
    for (int g = max(0, issued_k - C::NS); g < issued_k; ++g) drain_wait(&bar_k_full[g % C::NS], (g / C::NS) & 1);
    for (int g = max(0, issued_v - C::NS); g < issued_v; ++g) drain_wait(&bar_v_full[g % C::NS], (g / C::NS) & 1);
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
  if (a.Lq_seg > INT32_MAX - BM || a.Lk_seg > INT32_MAX - BN) return RATTN_ERR_UNSUPPORTED;
  if (a.nseg > kMaxHops) return RATTN_ERR_UNSUPPORTED;
  const int n_qtiles = static_cast<int>((a.Lq_seg + BM - 1) / BM);
  const long long grid = static_cast<long long>(a.BH) * a.nseg * n_qtiles;
  if (grid == 0) return RATTN_OK;
  if (grid > INT32_MAX) return RATTN_ERR_UNSUPPORTED;
  CUtensorMap tq, tk, tv;
  rattn_status st;
  if ((st = make_tmap_bf16(&tq, a.q, D, a.Lq_seg, a.nseg, a.BH, BM)) != RATTN_OK) return st;
  if (a.group < 1 || a.BH % a.group) return RATTN_ERR_INVALID_ARG;
  if ((st = make_tmap_bf16(&tk, a.k, D, a.Lk_seg, a.nseg, a.BH / a.group, BN)) != RATTN_OK) return st;
  if ((st = make_tmap_bf16(&tv, a.v, D, a.Lk_seg, a.nseg, a.BH / a.group, BN)) != RATTN_OK) return st;
  const void* kfn = a.seg ? reinterpret_cast<const void*>(&fwd_kernel<D, true>)
                         : reinterpret_cast<const void*>(&fwd_kernel<D, false>);
  if ((st = set_smem_attr(kfn, C::SMEM)) != RATTN_OK) return st;
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
    fwd_kernel<D, true><<<static_cast<unsigned>(grid), kThreads, C::SMEM, a.stream>>>(tq, tk, tv, p);
  else
    fwd_kernel<D, false><<<static_cast<unsigned>(grid), kThreads, C::SMEM, a.stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? RATTN_OK : RATTN_ERR_CUDA;
}

}  // namespace

// Forms of the bf16 forward (all compute the same attention; measured on B200):
//  - 256-key tiles (attn_fwd_wide_sm100.cu, D = 128, at most 32 segments): the
//    score product runs as N = 256 MMAs, about 1.6x the rate of N = 128 ones,
//    and the next score product overlaps the softmax; 4-8 % faster than the
//    other forms on dense rows of every length measured (16k to 1M keys);
//  - two 128-row query tiles per CTA (attn_fwd_pair_sm100.cu): half the K/V
//    bytes per FLOP; faster than one tile from 262,144 keys per row (where one
//    head's K and V outgrow L2), so the choice for long rows with D = 64;
//  - the persistent kernel (attn_fwd_persist_sm100.cu): work items of one
//    query tile taken from a per-launch counter; 8 % faster on packed
//    sequences, whose items are short, and slower per tile on dense rows;
//  - one 128-row query tile per CTA (this file): everything else.
// rattn_set_fwd_tiling forces one form (1 one tile, 2 two tiles, 3
// persistent, 4 256-key tiles).
constexpr long long kPairMinKeys = 262144;

rattn_status launch_fwd_sm100(const FwdArgs& a, const DevCtx& ctx) {
  switch (ctx.fwd_tiling) {
    case 1: break;
    case 2: return launch_fwd_sm100_pair(a, ctx);
    case 3: return launch_fwd_sm100_persist(a, ctx);
    case 4: return launch_fwd_sm100_wide(a, ctx);
    default:
      if (!a.seg && a.D == 128 && a.nseg <= 32) return launch_fwd_sm100_wide(a, ctx);
      if (static_cast<long long>(a.nseg) * a.Lk_seg >= kPairMinKeys) return launch_fwd_sm100_pair(a, ctx);
      if (a.seg) return launch_fwd_sm100_persist(a, ctx);
      break;
  }
  if (a.D == 128) return launch<128>(a, ctx);
  if (a.D == 64) return launch<64>(a, ctx);
  return RATTN_ERR_UNSUPPORTED;
}

}  // namespace rattn
