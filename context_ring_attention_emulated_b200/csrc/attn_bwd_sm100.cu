// attn_bwd_sm100.cu -- ring attention backward on the sm_100a tensor cores.
//
// Gradients of the ring forward ([CP-glossary] "Practical use and
// trade-offs" runs `.backward()` through the CP attention), recomputing the
// probabilities from the saved fp32 LSE instead of storing them:
//   P = exp(scale Q K^T - LSE),  dV = P^T dO,  dP = dO V^T,
//   dS = P o (dP - Delta),  Delta_i = dO_i . O_i,
//   dQ = scale dS K,  dK = scale dS^T Q.
// In a real ring the K/V block of rank s visits every rank r (at hop
// (r - s) mod cp) and its dK/dV travel with it; here one CTA keeps one
// 128-key K/V tile of rank s resident and walks every rank's query tiles in
// that hop order, skipping tiles the causal relation fully masks. dK and dV
// accumulate in TMEM. Each query tile's dQ contribution is read out of TMEM
// by a warpgroup of its own and added into an fp32 workspace by TMA tile
// reduce-adds from shared memory, which proceed in the background while the
// next tiles are computed; the workspace is converted to the output dtype at
// the end.
//
// Warp roles (512 threads):
//   warps 0..3   dQ read-out: one thread per query row; the whole dQ tile is
//                read out of TMEM into registers (freeing its columns at
//                once), then staged 128-byte swizzled in 32-column chunks,
//                one thread issuing the reduce-adds;
//   warps 4..11  two warpgroups, one thread per key row (TMEM lane) each:
//                P^T and dS^T over the warpgroup's 64 query columns, finally
//                half of dK/dV each;
//   warp 12      producer: K, V once; per query tile Q and dO by TMA and the
//                tile's LSE (pre-scaled by log2 e) and Delta into shared memory;
//   warp 13      TMEM allocation and tcgen05.mma issue (the whole warp walks
//                the schedule and waits, one lane chosen by elect.sync issues:
//                with the warp converged the operands stay warp-uniform; the
//                kernel ran about 20 % faster so than with a lone lane-0
//                thread walking the schedule);
//   warps 14, 15 idle (they complete the producer/MMA warpgroup, whose
//                registers the dQ warpgroup takes over: setmaxnreg).
// TMEM columns: [0,128) S^T, then P^T (bf16, warpgroup g at [64g, 64g+32));
// [128,256) dP^T, then dS^T (bf16, at 128 + [64g, 64g+32)), then dQ;
// dV [256,256+D); dK [256+D,256+2D). dS also goes to a swizzled shared tile,
// the A operand of dQ = dS K.
//
// Grouped key/value heads: the CTA of a K/V tile walks the query tiles of
// every query head of its group, so dK/dV sum over the group in TMEM. Packed
// sequences (the SEG instantiation): a key is visible only to queries with
// the same even segid; the producer flags per query tile whether any element
// needs masking.
//
// One hop across processes (the SPLIT instantiation, rattn_partial_bwd): the
// query rows belong to one rank and the key rows to another, so each side
// has its own length and position array; a single segment, no preparation
// pass (the caller hands in Delta and owns the fp32 dQ accumulator, which
// receives scale * dS K directly), and dK, dV leave as fp32 shares that are
// written or added to the caller's buffers.
#include <limits.h>
#include <math.h>

#include "debug_check.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace rattn {
namespace {

constexpr int kThreads = 512;  // 16 warps
constexpr int BQ = 128;        // query rows per tile
constexpr int BK = 128;        // key rows per CTA
constexpr int kMaxHops = 64;
constexpr int kWarpProducer = 12;
constexpr int kWarpMma = 13;
constexpr int kWarpCompute0 = 4;  // warps 4..11: two compute warpgroups
// Registers per thread: the kernel is launched with kLaunchRegs; the dQ
// warpgroup (warps 0..3) then grows to kRegsReduce, taken from the
// producer/MMA warpgroup (warps 12..15), which shrinks to kRegsLoad; the
// compute warpgroups keep kLaunchRegs. 144 + 2 x 128 + 112 = 4 x 128.
constexpr int kLaunchRegs = 128;
constexpr int kRegsReduce = 144;
constexpr int kRegsLoad = 112;
static_assert(kRegsReduce + 2 * kLaunchRegs + kRegsLoad == 4 * kLaunchRegs, "register split must balance");
constexpr int kReduceBar = 1;     // named barrier of the dQ warpgroup (warps 0..3)

template <int D>
struct Cfg {
  static constexpr int NSQ = 2;                   // Q stages (each with its LSE, Delta and mask flag)
  static constexpr int NSO = (D == 128) ? 1 : 2;  // dO stages
  static constexpr int TILE = 128 * D * 2;
  static constexpr int NBOX = D / 64;
  static constexpr int BOX = 128 * 128;           // one 128-row x 64-element box
  static constexpr int NCH = D / 32;              // 32-column chunks of a dQ tile
  static constexpr int CHUNK = 128 * 32 * 4;      // one staged fp32 dQ chunk
  static constexpr int NSTG = 2;                  // dQ staging buffers
  static constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 256 + D;
  static constexpr uint32_t T_COLS = 512;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;                 // NSQ stages
  static constexpr int OFF_DO = OFF_Q + NSQ * TILE;          // NSO stages
  static constexpr int OFF_DS = OFF_DO + NSO * TILE;         // 128 keys x 128 queries bf16, two boxes
  static constexpr int OFF_STG = OFF_DS + 2 * BOX;           // NSTG staged dQ chunks
  static constexpr int OFF_LSE = OFF_STG + NSTG * CHUNK;     // NSQ x 128 floats
  static constexpr int OFF_DELTA = OFF_LSE + NSQ * 128 * 4;  // NSQ x 128 floats
  static constexpr int OFF_BAR = OFF_DELTA + NSQ * 128 * 4;
  // barrier indices
  static constexpr int B_KV = 0, B_QF = 1, B_QE = B_QF + NSQ, B_OF = B_QE + NSQ, B_OE = B_OF + NSO,
                       B_SF = B_OE + NSO, B_PR = B_SF + 1, B_DPF = B_PR + 1, B_DSR = B_DPF + 1,
                       B_DQF = B_DSR + 1, B_DQE = B_DQF + 1, B_FIN = B_DQE + 1,
                       B_DRAIN = B_FIN + 1, NBAR = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_FULL = OFF_MISC + 16;  // NSQ ints: tile needs no masking
  static constexpr int OFF_HOP = OFF_FULL + 16;   // int2 table
  static constexpr int SMEM = OFF_HOP + kMaxHops * 8;
  static_assert(OFF_STG % 1024 == 0 && OFF_DS % 1024 == 0 && OFF_Q % 1024 == 0 && OFF_DO % 1024 == 0,
                "swizzled tiles need 1024-byte alignment");
  static_assert(OFF_HOP % 8 == 0 && OFF_BAR % 8 == 0 && NSQ <= 4, "shared-memory alignment");
  static_assert(SMEM <= 232448, "shared memory budget");
};

struct Params {
  const float* lse;
  const float* delta;
  const int32_t* pos;
  const int32_t* seg;  // packed sequences: segid per slot, or NULL
  int BH, group, nseg, Lseg, nq_tiles, nk_tiles, causal;
  long long kv_valid;
  float scale, scale_log2;
  void* dk;
  void* dv;
  int* err;
  unsigned long long wait_ns;
  // SPLIT only
  const int32_t* q_pos;   // query positions [Lq]
  const int32_t* kv_pos;  // key positions [Lk]
  int Lq, Lk;             // query and key rows (the ring uses Lseg for both)
  int accumulate;         // 1 adds the dK, dV shares to the outputs, 0 writes them
};

__device__ __forceinline__ int segat(const Params& p, int rank, int row) {
  const long long i = static_cast<long long>(rank) * p.Lseg + row;
  if (!in_bounds(i, static_cast<long long>(p.nseg) * p.Lseg, p.err, 11)) return 1;
  return __ldg(p.seg + i);
}

__device__ __forceinline__ long long posat(const Params& p, int seg, int row) {
  const long long i = static_cast<long long>(seg) * p.Lseg + row;
  if (!in_bounds(i, static_cast<long long>(p.nseg) * p.Lseg, p.err, 12)) return 0;
  return static_cast<long long>(__ldg(p.pos + i));
}

// Query-side and key-side lengths and positions: one array of Lseg rows per
// segment for the ring, separate arrays for a SPLIT hop.
template <bool SPLIT>
__device__ __forceinline__ int q_len(const Params& p) {
  return SPLIT ? p.Lq : p.Lseg;
}

template <bool SPLIT>
__device__ __forceinline__ int k_len(const Params& p) {
  return SPLIT ? p.Lk : p.Lseg;
}

template <bool SPLIT>
__device__ __forceinline__ long long qposat(const Params& p, int seg, int row) {
  if constexpr (SPLIT) {
    const long long i = static_cast<long long>(seg) * p.Lq + row;
    if (!in_bounds(i, p.Lq, p.err, 13)) return 0;
    return static_cast<long long>(__ldg(p.q_pos + i));
  } else {
    return posat(p, seg, row);
  }
}

template <bool SPLIT>
__device__ __forceinline__ long long kposat(const Params& p, int seg, int row) {
  if constexpr (SPLIT) {
    const long long i = static_cast<long long>(seg) * p.Lk + row;
    if (!in_bounds(i, p.Lk, p.err, 14)) return 0;
    return static_cast<long long>(__ldg(p.kv_pos + i));
  } else {
    return posat(p, seg, row);
  }
}

// The dQ warpgroup's hand-off of one 128-row x 32-column fp32 chunk (this
// thread's row in v) to the TMA: wait until the staging buffer's previous
// reduce-add has read it, write the row 128-byte swizzled (16-byte piece j of
// row r at piece j ^ (r mod 8): conflict-free for a warp's 32 rows), make the
// writes visible to the async proxy, and let one thread issue the tile
// reduce-add into the accumulator at (column c0, row r0) of segment `seg` of
// (batch, head) `bh`.
template <int D>
__device__ __forceinline__ void stage_dq_chunk(const uint32_t (&v)[32], uint8_t* buf, int row, bool elected,
                                               bool wait_buffer, const CUtensorMap* tm, int c0, int r0, int seg,
                                               int bh) {
  if (elected && wait_buffer) bulk_wait_group_read<Cfg<D>::NSTG - 1>();
  bar_sync(kReduceBar, 128);
  uint8_t* rowp = buf + row * 128;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    *reinterpret_cast<uint4*>(rowp + ((j ^ (row & 7)) << 4)) = make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2],
                                                                          v[4 * j + 3]);
  fence_proxy_async_smem();
  bar_sync(kReduceBar, 128);
  if (elected) {
    tma_reduce_add_4d(tm, buf, c0, r0, seg, bh);
    bulk_commit_group();
  }
}

// 16 warps share an SM's four register-file partitions 4/4/4/4: 16,384 / (4 x
// 32) = 128 registers per thread at launch.
// SEG: packed sequences; SPLIT: one hop across processes; DQ = false: dK and
// dV only (the deterministic mode forms dQ in a query-stationary pass).
template <int D, bool SEG, bool SPLIT, bool DQ = true>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
               const __grid_constant__ CUtensorMap tm_dq, const Params p) {
  using C = Cfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* bar_kv_full = bars + C::B_KV;
  uint64_t* bar_q_full = bars + C::B_QF;
  uint64_t* bar_q_empty = bars + C::B_QE;
  uint64_t* bar_o_full = bars + C::B_OF;
  uint64_t* bar_o_empty = bars + C::B_OE;
  uint64_t* bar_s_full = bars + C::B_SF;      // S^T(j) in TMEM
  uint64_t* bar_p_ready = bars + C::B_PR;     // P^T(j) written over it (one arrival per compute warp)
  uint64_t* bar_dp_full = bars + C::B_DPF;    // dP^T(j) in TMEM
  uint64_t* bar_ds_ready = bars + C::B_DSR;   // dS^T(j) over dP^T(j) and dS(j) in shared memory
  uint64_t* bar_dq_full = bars + C::B_DQF;    // dQ(j) in TMEM (dS(j) in shared memory consumed)
  uint64_t* bar_dq_empty = bars + C::B_DQE;   // dQ(j) read out of TMEM (one arrival per dQ warp)
  uint64_t* bar_fin = bars + C::B_FIN;        // every MMA completed
  uint64_t* bar_drain = bars + C::B_DRAIN;

  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  // per hop: x = first visible query tile; y = end of the visible tiles for
  // packed sequences, else the first tile with no masked element (the visible
  // tiles then run to the last tile)
  int2* s_hop = reinterpret_cast<int2*>(smem + C::OFF_HOP);
  volatile int* s_full = reinterpret_cast<volatile int*>(smem + C::OFF_FULL);  // per Q stage
  float* s_lse = reinterpret_cast<float*>(smem + C::OFF_LSE);
  float* s_delta = reinterpret_cast<float*>(smem + C::OFF_DELTA);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // The 128-byte swizzle needs 1024-byte aligned tiles; refuse to run otherwise.
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0 && p.err) atomicCAS(p.err, 0, SITE_BWD_LOAD);
    return;
  }

  // Work item: (batch, head) slowest, so the CTAs resident at any time share
  // one head's Q, dO and dQ accumulator in L2; within a head the key tiles
  // with the smallest positions (seen by the most queries) go first.
  int item = blockIdx.x;
  const int s = item % p.nseg;
  item /= p.nseg;
  const int kt = item % p.nk_tiles;
  const int kvh = item / p.nk_tiles;  // (batch, key/value head); its query heads are kvh * group + j
  const int k0 = kt * BK;
  const int k_rows = min(BK, k_len<SPLIT>(p) - k0);
  const long long k_min = kposat<SPLIT>(p, s, k0);
  const long long k_max = kposat<SPLIT>(p, s, k0 + k_rows - 1);

  if (threadIdx.x == 0) {
    mbar_init(bar_kv_full, 1);
    for (int i = 0; i < C::NSQ; ++i) {
      mbar_init(&bar_q_full[i], 1);
      mbar_init(&bar_q_empty[i], 1);
    }
    for (int i = 0; i < C::NSO; ++i) {
      mbar_init(&bar_o_full[i], 1);
      mbar_init(&bar_o_empty[i], 1);
    }
    mbar_init(bar_s_full, 1);
    mbar_init(bar_p_ready, 8);
    mbar_init(bar_dp_full, 1);
    mbar_init(bar_ds_ready, 8);
    mbar_init(bar_dq_full, 1);
    mbar_init(bar_dq_empty, 4);
    mbar_init(bar_fin, 1);
    mbar_init(bar_drain, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) tmem_alloc(s_tmem, C::T_COLS);

  // Per hop t the query segment is r = (s + t) mod nseg. Visible query tiles
  // form a range [first_vis, end_vis): positions (and segids for packed
  // sequences) are non-decreasing in a segment, so both ends are partition
  // points of predicates that hold on a prefix (one warp per hop, 32-way
  // searches); without packed sequences end_vis = nq_tiles.
  const bool live = k_min < p.kv_valid;
  const int sk_lo = SEG ? segat(p, s, k0) : 0;
  const int sk_hi = SEG ? segat(p, s, k0 + k_rows - 1) : 0;
  for (int t = warp; t < p.nseg; t += kThreads / 32) {
    const int r = (s + t) % p.nseg;
    int first_vis = p.nq_tiles, end_vis = p.nq_tiles;
    if (live) {
      first_vis = warp_partition_point(0, p.nq_tiles, lane, [&](int m) {  // last query sees no key of this tile
        const int last = min((m + 1) * BQ, q_len<SPLIT>(p)) - 1;
        return !((!p.causal || qposat<SPLIT>(p, r, last) >= k_min) && (!SEG || segat(p, r, last) >= sk_lo));
      });
      if (SEG)  // up to the first tile wholly past the key tile's last segment
        end_vis = warp_partition_point(first_vis, p.nq_tiles, lane, [&](int m) { return segat(p, r, m * BQ) <= sk_hi; });
      else if (p.causal)  // up to the first tile whose first query sees every key
        end_vis = warp_partition_point(first_vis, p.nq_tiles, lane,
                                       [&](int m) { return qposat<SPLIT>(p, r, m * BQ) < k_max; });
      else
        end_vis = first_vis;  // non-causal: every visible tile is unmasked
    }
    if (lane == 0) s_hop[t] = make_int2(first_vis, end_vis);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  int NIT = 0;
  for (int t = 0; t < p.nseg; ++t) NIT += (SEG ? s_hop[t].y : p.nq_tiles) - s_hop[t].x;
  NIT *= p.group;  // the same tiles for every query head of the group

  int issued_q = 0, issued_o = 0;
  bool kv_issued = false;

  if (warp >= kWarpProducer) {
    regs_dec<kRegsLoad>();  // warps 12..15 (14 and 15 idle)
  if (warp == kWarpProducer) {
    // ------------------------------------------------------------ producer
    if (NIT > 0) {
      if (lane == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(&tm_do);
        mbar_arrive_expect_tx(bar_kv_full, 2 * C::TILE);
        for (int b = 0; b < C::NBOX; ++b) {
          tma_load_4d(smem + C::OFF_K + b * C::BOX, &tm_k, bar_kv_full, b * 64, k0, s, kvh);
          tma_load_4d(smem + C::OFF_V + b * C::BOX, &tm_v, bar_kv_full, b * 64, k0, s, kvh);
        }
      }
      kv_issued = true;
      bool ok = true;
      int it = 0;
      for (int hq = 0; hq < p.group && ok; ++hq) {
      const int bh = kvh * p.group + hq;  // (batch, query head)
      for (int t = 0; t < p.nseg && ok; ++t) {
        const int r = (s + t) % p.nseg;
        const int i_end = SEG ? s_hop[t].y : p.nq_tiles;
        for (int i = s_hop[t].x; i < i_end; ++i, ++it) {
          const int st = it % C::NSQ;
          const uint32_t u = it / C::NSQ;
          if (u > 0 && !warp_wait(&bar_q_empty[st], (u - 1) & 1, s_abort, p.wait_ns)) {
            if (lane == 0) record_failure(s_abort, p.err, SITE_BWD_LOAD);
            ok = false;
            break;
          }
          const long long rowbase = (static_cast<long long>(bh) * p.nseg + r) * q_len<SPLIT>(p);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = e * 32 + lane;  // coalesced loads, conflict-free stores
            const int q = i * BQ + c;
            float l2 = INFINITY, dl = 0.f;
            if (q < q_len<SPLIT>(p) &&
                in_bounds(rowbase + q, static_cast<long long>(p.BH) * p.nseg * q_len<SPLIT>(p), p.err, 15)) {
              const float l = __ldg(p.lse + rowbase + q);
              l2 = l == -INFINITY ? INFINITY : l * 1.4426950408889634f;
              dl = __ldg(p.delta + rowbase + q);
            }
            s_lse[st * 128 + c] = l2;
            s_delta[st * 128 + c] = dl;
          }
          if (lane == 0) {
            // No element of this tile pair is masked when every query sees
            // every key. Without packed sequences that is the tiles from the
            // hop table's y on; packed, all in one real sequence and, when
            // causal, the first query at or after the last key.
            bool full = i >= s_hop[t].y;
            if (SEG) {
              const int qa = i * BQ, qb = min(qa + BQ, q_len<SPLIT>(p)) - 1;
              full = (!p.causal || qposat<SPLIT>(p, r, qa) >= k_max) && sk_lo == sk_hi && (sk_lo & 1) == 0 &&
                     segat(p, r, qa) == sk_lo && segat(p, r, qb) == sk_lo;
            }
            s_full[st] = full ? 1 : 0;
          }
          __syncwarp();
          if (elect_one()) {
            mbar_arrive_expect_tx(&bar_q_full[st], C::TILE);
            for (int b = 0; b < C::NBOX; ++b)
              tma_load_4d(smem + C::OFF_Q + st * C::TILE + b * C::BOX, &tm_q, &bar_q_full[st], b * 64, i * BQ, r,
                          bh);
          }
          ++issued_q;
          const int so = it % C::NSO;
          const uint32_t uo = it / C::NSO;
          if (uo > 0 && !warp_wait(&bar_o_empty[so], (uo - 1) & 1, s_abort, p.wait_ns)) {
            if (lane == 0) record_failure(s_abort, p.err, SITE_BWD_LOAD);
            ok = false;
            break;
          }
          if (elect_one()) {
            mbar_arrive_expect_tx(&bar_o_full[so], C::TILE);
            for (int b = 0; b < C::NBOX; ++b)
              tma_load_4d(smem + C::OFF_DO + so * C::TILE + b * C::BOX, &tm_do, &bar_o_full[so], b * 64, i * BQ,
                          r, bh);
          }
          ++issued_o;
        }
      }
      }
    }
  } else if (warp == kWarpMma) {
    // ----------------------------------------------------------- MMA issue
    // Per query tile j: S^T(j) = K Q^T, dP^T(j) = V dO^T, dV += P^T dO,
    // dK += dS^T Q (dS^T read from TMEM over dP^T), dQ(j) = dS K (into the
    // dP^T columns). Issue order, steady state:
    //   dK(i), dQ(i), dP(i+1), dV(i+1), S(i+2)
    // dP(i+1) is on the chain dS(i) -> dK / dQ(i) -> read-out of dQ(i) ->
    // dP(i+1) -> dS(i+1), so it goes first once dQ(i) is out of TMEM; dV and
    // S fill the pipe while the compute warpgroups form dS(i+1). MMAs issued
    // by one thread execute in issue order, so dQ(i) follows dK(i) without a
    // wait although it overwrites the dS^T columns dK(i) reads, and S(j)
    // follows dV(j-1), which reads the P^T columns S(j) overwrites.
    if (NIT > 0) {  // the whole warp walks the schedule and waits; one elected lane issues
      const uint32_t idesc_t = idesc_bf16_f32(BK, BQ, 0, 0);  // S^T, dP^T: K-major A and B
      const uint32_t idesc_g = idesc_bf16_f32(BK, D, 0, 1);   // dV, dK: A in TMEM, B MN-major
      const uint32_t idesc_q = idesc_bf16_f32(BQ, D, 1, 1);   // dQ: A (dS) and B (K) MN-major
      // Operand descriptors as one base descriptor per layout plus byte offsets.
      const uint64_t dk_s = sdesc_sw128(smem_u32(smem), 16, 1024);      // K-major tiles
      const uint64_t dmn = sdesc_sw128(smem_u32(smem), C::BOX, 1024);   // MN-major tiles
      auto oQ = [&](int j) { return static_cast<uint32_t>(C::OFF_Q + (j % C::NSQ) * C::TILE); };
      auto oDO = [&](int j) { return static_cast<uint32_t>(C::OFF_DO + (j % C::NSO) * C::TILE); };
      auto wt = [&](uint64_t* bar, uint32_t parity) { return warp_wait(bar, parity, s_abort, p.wait_ns); };

      auto mma_s = [&](int j) -> bool {
        if (!wt(&bar_q_full[j % C::NSQ], (j / C::NSQ) & 1)) return false;
        tc_fence_after();
        if (elect_one()) {
          const uint32_t q = oQ(j);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
            umma_ss(tmem + C::T_S, sdesc_add(dk_s, C::OFF_K + off), sdesc_add(dk_s, q + off), idesc_t,
                    kk > 0 ? 1u : 0u);
          }
          umma_commit(bar_s_full);
        }
        __syncwarp();
        return true;
      };
      auto mma_dp = [&](int j) -> bool {
        if (!wt(&bar_o_full[j % C::NSO], (j / C::NSO) & 1)) return false;
        if constexpr (DQ) {
          if (j > 0 && !wt(bar_dq_empty, (j - 1) & 1)) return false;  // dQ(j-1) read out
        } else {  // dK(j-1), the last reader of dS^T(j-1), has completed
          if (j > 0 && !wt(&bar_q_empty[(j - 1) % C::NSQ], ((j - 1) / C::NSQ) & 1)) return false;
        }
        tc_fence_after();
        if (elect_one()) {
          const uint32_t o = oDO(j);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::BOX + (kk & 3) * 32;
            umma_ss(tmem + C::T_DP, sdesc_add(dk_s, C::OFF_V + off), sdesc_add(dk_s, o + off), idesc_t,
                    kk > 0 ? 1u : 0u);
          }
          umma_commit(bar_dp_full);
          if (j == 0) umma_commit(&bar_o_empty[0]);  // dV(0) was issued before dP(0)
        }
        __syncwarp();
        return true;
      };
      auto mma_dv = [&](int j) -> bool {
        if (!wt(bar_p_ready, j & 1)) return false;
        if (!wt(&bar_o_full[j % C::NSO], (j / C::NSO) & 1)) return false;
        tc_fence_after();
        if (elect_one()) {
          const uint32_t o = oDO(j);
#pragma unroll
          for (int kk = 0; kk < BQ / 16; ++kk) {
            const uint32_t a_col = C::T_S + (kk >> 2) * 64 + (kk & 3) * 8;  // warpgroup (kk >> 2)'s P^T
            umma_ts(tmem + C::T_DV, tmem + a_col, sdesc_add(dmn, o + kk * 2048), idesc_g,
                    (j > 0 || kk > 0) ? 1u : 0u);
          }
          if (j > 0) umma_commit(&bar_o_empty[j % C::NSO]);  // dP(j) was issued before dV(j)
        }
        __syncwarp();
        return true;
      };
      auto mma_dk = [&](int j) -> bool {
        if (!wt(bar_ds_ready, j & 1)) return false;
        tc_fence_after();
        if (elect_one()) {
          const uint32_t q = oQ(j);
#pragma unroll
          for (int kk = 0; kk < BQ / 16; ++kk) {
            const uint32_t a_col = C::T_DP + (kk >> 2) * 64 + (kk & 3) * 8;  // warpgroup (kk >> 2)'s dS^T
            umma_ts(tmem + C::T_DK, tmem + a_col, sdesc_add(dmn, q + kk * 2048), idesc_g,
                    (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bar_q_empty[j % C::NSQ]);  // S(j) and dK(j) were Q's readers
        }
        __syncwarp();
        return true;
      };
      auto mma_dq = [&](int j) -> bool {
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_ss(tmem + C::T_DP, sdesc_add(dmn, C::OFF_DS + kk * 2048), sdesc_add(dmn, C::OFF_K + kk * 2048),
                    idesc_q, kk > 0 ? 1u : 0u);
          umma_commit(bar_dq_full);
        }
        __syncwarp();
        return true;
      };

      bool ok = wt(bar_kv_full, 0);
      ok = ok && mma_s(0) && mma_dv(0) && mma_dp(0) && (NIT < 2 || mma_s(1));
      for (int i = 0; i < NIT && ok; ++i) {
        ok = mma_dk(i) && (!DQ || mma_dq(i));
        if (ok && i + 1 < NIT) ok = mma_dp(i + 1) && mma_dv(i + 1);
        if (ok && i + 2 < NIT) ok = mma_s(i + 2);
      }
      if (ok) {
        if (elect_one()) umma_commit(bar_fin);
        __syncwarp();
      } else if (lane == 0) {
        record_failure(s_abort, p.err, SITE_BWD_MMA);
      }
    }
  }
  } else if (warp >= kWarpCompute0) {
    // ------------------------------------------------- P^T and dS^T per key
    // Two warpgroups; warpgroup wg owns query columns [64 wg, 64 wg + 64) of
    // every tile (and D columns [wg D/2, (wg+1) D/2) of dK, dV at the end).
    // Each writes P^T / dS^T only into TMEM columns it alone has read: P^T of
    // its columns at T_S + 64 wg, dS^T at T_DP + 64 wg (bf16 pairs).
    const int wg = (warp - kWarpCompute0) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // key row
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const bool key_ok = row < k_rows;
    const long long my_kpos = key_ok ? kposat<SPLIT>(p, s, k0 + row) : k_max;
    if (kDebugChecks && wg == 0 && key_ok && k0 + row > 0)
      check_order(kposat<SPLIT>(p, s, k0 + row - 1) <= my_kpos, p.err, 18);
    const int my_seg = (SEG && key_ok) ? segat(p, s, k0 + row) : 0;
    const bool key_dead = !key_ok || my_kpos >= p.kv_valid || (my_seg & 1);  // odd segid: padding
    const float sl2 = p.scale_log2;
    const int qc0 = wg * 64;  // first query column of this warpgroup
    const uint32_t t_s = tmem + lane_base + C::T_S + qc0;
    const uint32_t t_dp = tmem + lane_base + C::T_DP + qc0;
    uint8_t* sds = smem + C::OFF_DS + wg * C::BOX;
    bool ok = true;
    int it = 0;
    for (int hq = 0; hq < p.group && ok; ++hq) {
    for (int t = 0; t < p.nseg && ok; ++t) {
      const int r = (s + t) % p.nseg;
      const int i_end = SEG ? s_hop[t].y : p.nq_tiles;
      for (int i = s_hop[t].x; i < i_end; ++i, ++it) {
        const int st = it % C::NSQ;
        const float* lse2 = s_lse + st * 128 + qc0;
        const float* dlt = s_delta + st * 128 + qc0;
        // Query columns of this tile that see this key: [first, last). The
        // tile's query positions (and segids when packed) are spread over
        // the warp, four per lane, read with one coalesced load before the
        // wait for the tile's scores; every lane then finds its key's bounds
        // by binary search through shuffles (eight steps cover 128 queries;
        // all lanes take every step). Only tiles with a masked element need
        // it: without packed sequences the hop table says which, packed the
        // producer's flag does.
        int first = 0, last = BQ;
        const int n = min(BQ, q_len<SPLIT>(p) - i * BQ);
        int qp4[4], qs4[4];
        auto load_tile_keys = [&]() {
          const long long qbase = static_cast<long long>(r) * q_len<SPLIT>(p) + i * BQ;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int idx = 4 * lane + e;
            const bool inb = idx < n && in_bounds(qbase + idx, static_cast<long long>(p.nseg) * q_len<SPLIT>(p), p.err, 16);
            qp4[e] = inb ? __ldg((SPLIT ? p.q_pos : p.pos) + qbase + idx) : INT_MAX;
            qs4[e] = (SEG && inb) ? __ldg(p.seg + qbase + idx) : INT_MAX;
          }
        };
        auto search = [&]() {
          int lo = 0, hi = n;
#pragma unroll 1
          for (int step = 0; step < 8; ++step) {  // first query at or after this key (same sequence when packed)
            const int mid = (lo + hi) >> 1;
            const int qp = warp_elem128(qp4, mid);
            const int qs = SEG ? warp_elem128(qs4, mid) : 0;
            const bool past = p.causal ? qp >= my_kpos : (!SEG || qs >= my_seg);
            if (lo < hi) {
              if (past) hi = mid; else lo = mid + 1;
            }
          }
          first = lo;
          if (SEG) {
            hi = n;
#pragma unroll 1
            for (int step = 0; step < 8; ++step) {  // first query of a later sequence
              const int mid = (lo + hi) >> 1;
              const int qs = warp_elem128(qs4, mid);
              if (lo < hi) {
                if (qs > my_seg) hi = mid; else lo = mid + 1;
              }
            }
            last = lo;
          }
        };
        // Without packed sequences only tiles before the hop table's y hold
        // masked elements (the same for the whole warp).
        const bool unpacked_masked = !SEG && i < s_hop[t].y;
        if (unpacked_masked) load_tile_keys();
        if (!warp_wait(&bar_q_full[st], (it / C::NSQ) & 1, s_abort, p.wait_ns)) {
          if (lane == 0) record_failure(s_abort, p.err, SITE_BWD_COMPUTE);
          ok = false;
          break;
        }
        const bool packed_masked = SEG && !s_full[st];  // the same for the whole warp
        if (packed_masked) load_tile_keys();
        if (!warp_wait(bar_s_full, it & 1, s_abort, p.wait_ns)) {
          if (lane == 0) record_failure(s_abort, p.err, SITE_BWD_COMPUTE);
          ok = false;
          break;
        }
        tc_fence_after();
        if (unpacked_masked || packed_masked) search();
        if (key_dead) first = BQ;
        first -= qc0;  // relative to this warpgroup's columns
        last -= qc0;
        uint32_t sr[2][32];
        tmem_ld32(t_s, sr[0]);
        tmem_ld32(t_s + 32, sr[1]);
        tmem_wait_ld();
        // P^T (fp32, kept in sr) and its bf16 copy over its scores, 32 query
        // columns at a time
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c0 = 32 * h + 2 * e;
            float a = ex2_approx(fmaf(__uint_as_float(sr[h][2 * e]), sl2, -lse2[c0]));
            float b = ex2_approx(fmaf(__uint_as_float(sr[h][2 * e + 1]), sl2, -lse2[c0 + 1]));
            if (SEG) {  // visible run [first, last)
              a = (c0 >= first && c0 < last) ? a : 0.f;
              b = (c0 + 1 >= first && c0 + 1 < last) ? b : 0.f;
            } else {      // visible suffix from first
              a = c0 >= first ? a : 0.f;
              b = c0 + 1 >= first ? b : 0.f;
            }
            sr[h][2 * e] = __float_as_uint(a);
            sr[h][2 * e + 1] = __float_as_uint(b);
            pk[e] = pack_bf16x2(a, b);
          }
          tmem_st16(t_s + 16 * h, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_p_ready);  // one arrival per warp
        // dS(j) goes into the shared tile that dQ(j-1) reads: wait for it.
        if (!warp_wait(bar_dp_full, it & 1, s_abort, p.wait_ns) ||
            (DQ && it > 0 && !warp_wait(bar_dq_full, (it - 1) & 1, s_abort, p.wait_ns))) {
          if (lane == 0) record_failure(s_abort, p.err, SITE_BWD_COMPUTE);
          ok = false;
          break;
        }
        tc_fence_after();
        // dS^T = P^T o (dP^T - Delta): bf16 over this warpgroup's dP^T
        // columns in TMEM (read by dK) and into the swizzled shared tile read
        // by dQ (box wg, row = key), 16 query columns at a time (the packed
        // pairs of chunk c land on columns already read).
        uint8_t* rowp = sds + row * 128;
        uint32_t dpb[2][16];  // chunk c in dpb[c & 1]; chunk c + 1 is read while c is processed
        tmem_ld16(t_dp, dpb[0]);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tmem_wait_ld();
          if (c + 1 < 4) tmem_ld16(t_dp + (c + 1) * 16, dpb[(c + 1) & 1]);
          const uint32_t (&dp)[16] = dpb[c & 1];
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int q0 = c * 16 + 2 * e;
            const float a = __uint_as_float(sr[c >> 1][(c & 1) * 16 + 2 * e]) * (__uint_as_float(dp[2 * e]) - dlt[q0]);
            const float b =
                __uint_as_float(sr[c >> 1][(c & 1) * 16 + 2 * e + 1]) * (__uint_as_float(dp[2 * e + 1]) - dlt[q0 + 1]);
            pk[e] = pack_bf16x2(a, b);
          }
          tmem_st8(t_dp + c * 8, pk);
          if constexpr (DQ) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int chunk = c * 2 + j;
              *reinterpret_cast<uint4*>(rowp + ((chunk ^ (row & 7)) << 4)) =
                  make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
            }
          }
        }
        tmem_wait_st();
        if constexpr (DQ) fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_ds_ready);  // one arrival per warp
      }
    }
    }
    // ------------------------------------------------------ dK, dV out
    if (ok && NIT > 0 && !warp_wait(bar_fin, 0, s_abort, p.wait_ns)) {
      if (lane == 0) record_failure(s_abort, p.err, SITE_BWD_EPILOGUE);
      ok = false;
    }
    if (ok) {
      if (NIT > 0) tc_fence_after();
      const long long krow = (static_cast<long long>(kvh) * p.nseg + s) * k_len<SPLIT>(p) + k0 + row;
      const bool out_ok =
          !key_ok || in_bounds(krow, static_cast<long long>(p.BH / p.group) * p.nseg * k_len<SPLIT>(p), p.err, 17);
      __nv_bfloat16* dk = static_cast<__nv_bfloat16*>(p.dk) + krow * D + wg * (D / 2);
      __nv_bfloat16* dv = static_cast<__nv_bfloat16*>(p.dv) + krow * D + wg * (D / 2);
      float* dk32 = static_cast<float*>(p.dk) + krow * D + wg * (D / 2);
      float* dv32 = static_cast<float*>(p.dv) + krow * D + wg * (D / 2);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t gk[32], gv[32];
        if (NIT > 0) {
          tmem_ld32(tmem + lane_base + C::T_DK + wg * (D / 2) + c * 32, gk);
          tmem_ld32(tmem + lane_base + C::T_DV + wg * (D / 2) + c * 32, gv);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) gk[e] = gv[e] = 0u;
        }
        if (SPLIT && key_ok && out_ok) {  // fp32 shares, written or added (this thread owns these elements)
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float4 wk = make_float4(__uint_as_float(gk[4 * e + 0]) * p.scale, __uint_as_float(gk[4 * e + 1]) * p.scale,
                                    __uint_as_float(gk[4 * e + 2]) * p.scale, __uint_as_float(gk[4 * e + 3]) * p.scale);
            float4 wv = make_float4(__uint_as_float(gv[4 * e + 0]), __uint_as_float(gv[4 * e + 1]),
                                    __uint_as_float(gv[4 * e + 2]), __uint_as_float(gv[4 * e + 3]));
            float4* pk = reinterpret_cast<float4*>(dk32 + c * 32) + e;
            float4* pv = reinterpret_cast<float4*>(dv32 + c * 32) + e;
            if (p.accumulate) {
              const float4 ok4 = *pk, ov4 = *pv;
              wk.x += ok4.x; wk.y += ok4.y; wk.z += ok4.z; wk.w += ok4.w;
              wv.x += ov4.x; wv.y += ov4.y; wv.z += ov4.z; wv.w += ov4.w;
            }
            *pk = wk;
            *pv = wv;
          }
        } else if (key_ok && out_ok) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint4 wk, wv;
            wk.x = pack_bf16x2(__uint_as_float(gk[8 * e + 0]) * p.scale, __uint_as_float(gk[8 * e + 1]) * p.scale);
            wk.y = pack_bf16x2(__uint_as_float(gk[8 * e + 2]) * p.scale, __uint_as_float(gk[8 * e + 3]) * p.scale);
            wk.z = pack_bf16x2(__uint_as_float(gk[8 * e + 4]) * p.scale, __uint_as_float(gk[8 * e + 5]) * p.scale);
            wk.w = pack_bf16x2(__uint_as_float(gk[8 * e + 6]) * p.scale, __uint_as_float(gk[8 * e + 7]) * p.scale);
            wv.x = pack_bf16x2(__uint_as_float(gv[8 * e + 0]), __uint_as_float(gv[8 * e + 1]));
            wv.y = pack_bf16x2(__uint_as_float(gv[8 * e + 2]), __uint_as_float(gv[8 * e + 3]));
            wv.z = pack_bf16x2(__uint_as_float(gv[8 * e + 4]), __uint_as_float(gv[8 * e + 5]));
            wv.w = pack_bf16x2(__uint_as_float(gv[8 * e + 6]), __uint_as_float(gv[8 * e + 7]));
            reinterpret_cast<uint4*>(dk + c * 32)[e] = wk;
            reinterpret_cast<uint4*>(dv + c * 32)[e] = wv;
          }
        }
      }
    }
  } else {
    regs_inc<kRegsReduce>();
    // ------------------------------------------------------ dQ read-out
    // Warps 0..3, one thread per query row (TMEM lane): each dQ(j) is read
    // out of TMEM whole (D registers per thread), which releases the dP^T
    // columns at once; then it is staged in shared memory in 32-column
    // chunks and added into the fp32 accumulator by TMA tile reduce-adds,
    // which run on in the background while the next tiles are computed. One
    // thread issues the copies; named barriers keep the warpgroup in step,
    // and every decision to stop is taken together (so no thread is left at
    // a barrier).
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // query row
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const bool elected = threadIdx.x == 0;
    uint8_t* stg = smem + C::OFF_STG;
    int n_staged = 0;
    bool ok = DQ && NIT > 0;
    int it = 0;
    for (int hq = 0; hq < p.group && ok; ++hq) {
    const int bh = kvh * p.group + hq;  // (batch, query head)
    for (int t = 0; t < p.nseg && ok; ++t) {
      const int r = (s + t) % p.nseg;
      const int i_end = SEG ? s_hop[t].y : p.nq_tiles;
      for (int i = s_hop[t].x; i < i_end; ++i, ++it) {
        const bool got = mbar_wait(bar_dq_full, it & 1, s_abort, p.wait_ns);
        if (bar_any(kReduceBar, 128, !got)) {
          if (elected) record_failure(s_abort, p.err, SITE_BWD_COMPUTE);
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t v[C::NCH][32];
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) tmem_ld32(tmem + lane_base + C::T_DP + c * 32, v[c]);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_dq_empty);  // one arrival per warp
        if constexpr (SPLIT) {  // the caller's accumulator holds dQ itself
#pragma unroll
          for (int c = 0; c < C::NCH; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e) v[c][e] = __float_as_uint(__uint_as_float(v[c][e]) * p.scale);
        }
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          stage_dq_chunk<D>(v[c], stg + (n_staged % C::NSTG) * C::CHUNK, row, elected, n_staged >= C::NSTG, &tm_dq,
                            c * 32, i * BQ, r, bh);
          ++n_staged;
        }
      }
    }
    }
    if (elected) bulk_wait_all();  // the staged chunks are read before shared memory goes away
  }

  // ------------------------------------------------------------ teardown
  if (warp == kWarpProducer && lane == 0) {
    if (kv_issued) drain_wait(bar_kv_full, 0);
    for (int it = max(0, issued_q - C::NSQ); it < issued_q; ++it)
      drain_wait(&bar_q_full[it % C::NSQ], (it / C::NSQ) & 1);
    for (int it = max(0, issued_o - C::NSO); it < issued_o; ++it)
      drain_wait(&bar_o_full[it % C::NSO], (it / C::NSO) & 1);
  }
  if (warp == kWarpMma && NIT > 0) {  // the lane that issued the products commits
    if (elect_one()) {
      umma_commit(bar_drain);
      if (!drain_wait(bar_drain, 0)) record_failure(s_abort, p.err, SITE_DRAIN);
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::T_COLS);
  }
}

// Delta_i = dO_i . O_i (fp32) and (ZERO_DQ) zeroing of the dQ accumulator
// rows: one 16-lane group per row, 16-byte loads.
template <int D, bool ZERO_DQ>
__global__ void bwd_prep_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                                float* __restrict__ delta, float* __restrict__ dq_acc, long long rows) {
  constexpr int V = D / 8;  // 16-byte vectors per bf16 row
  const long long gid = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  const long long row = gid / 16;
  const int l = static_cast<int>(gid & 15);
  float s = 0.f;
  if (row < rows) {
    for (int e = l; e < V; e += 16) {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(o + row * D) + e);
      const uint4 b = __ldg(reinterpret_cast<const uint4*>(dout + row * D) + e);
      const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 fa = __bfloat1622float2(pa[j]);
        const float2 fb = __bfloat1622float2(pb[j]);
        s = fmaf(fa.x, fb.x, s);
        s = fmaf(fa.y, fb.y, s);
      }
    }
    if constexpr (ZERO_DQ) {
      float4* z = reinterpret_cast<float4*>(dq_acc + row * D);
      for (int e = l; e < D / 4; e += 16) z[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (row < rows && l == 0) delta[row] = s;
}

// dq = bf16(scale * dq_acc)
__global__ void dq_convert_kernel(const float4* __restrict__ acc, uint2* __restrict__ dq, float scale,
                                  long long n4) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 a = __ldg(acc + i);
    dq[i] = make_uint2(pack_bf16x2(a.x * scale, a.y * scale), pack_bf16x2(a.z * scale, a.w * scale));
  }
}

unsigned grid_for(long long work, int threads) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (work + threads - 1) / threads;
  const long long cap = static_cast<long long>(sms) * 16;
  return static_cast<unsigned>(want < cap ? (want > 0 ? want : 1) : cap);
}

// The register split among the warpgroups balances only if the kernel is
// launched with exactly kLaunchRegs per thread (a lower count would leave the
// dQ warpgroup's increase waiting for registers that never come): refuse to
// launch otherwise.
rattn_status check_launch_regs(const void* kfn) {
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kfn) != cudaSuccess) return RATTN_ERR_CUDA;
  return fa.numRegs == kLaunchRegs ? RATTN_OK : RATTN_ERR_UNSUPPORTED;
}

template <int D>
rattn_status launch(const BwdArgs& a, const DevCtx& ctx) {
  using C = Cfg<D>;
  if (a.Lseg > INT32_MAX - BQ || a.nseg > kMaxHops) return RATTN_ERR_UNSUPPORTED;
  const long long rows = static_cast<long long>(a.BH) * a.nseg * a.Lseg;
  const int nt = static_cast<int>((a.Lseg + 127) / 128);
  if (a.group < 1 || a.BH % a.group) return RATTN_ERR_INVALID_ARG;
  const long long grid = static_cast<long long>(a.BH / a.group) * a.nseg * nt;  // one CTA per key/value tile
  if (grid == 0) return RATTN_OK;
  if (grid > INT32_MAX) return RATTN_ERR_UNSUPPORTED;
  // Everything that can fail on the host comes before the first launch.
  CUtensorMap tq, tk, tv, tdo, tdq;
  rattn_status st;
  if ((st = make_tmap_bf16(&tq, a.q, D, a.Lseg, a.nseg, a.BH, BQ)) != RATTN_OK) return st;
  if ((st = make_tmap_bf16(&tk, a.k, D, a.Lseg, a.nseg, a.BH / a.group, BK)) != RATTN_OK) return st;
  if ((st = make_tmap_bf16(&tv, a.v, D, a.Lseg, a.nseg, a.BH / a.group, BK)) != RATTN_OK) return st;
  if ((st = make_tmap_bf16(&tdo, a.dout, D, a.Lseg, a.nseg, a.BH, BQ)) != RATTN_OK) return st;
  if ((st = make_tmap_f32_acc(&tdq, a.dq_acc, D, a.Lseg, a.nseg, a.BH)) != RATTN_OK) return st;
  // Deterministic mode: this kernel forms dK and dV only, and a
  // query-stationary pass forms dQ (no accumulator to zero or convert).
  const bool det = ctx.bwd_deterministic != 0;
  const void* kfn = det ? (a.seg ? reinterpret_cast<const void*>(&bwd_kernel<D, true, false, false>)
                                 : reinterpret_cast<const void*>(&bwd_kernel<D, false, false, false>))
                        : (a.seg ? reinterpret_cast<const void*>(&bwd_kernel<D, true, false>)
                                 : reinterpret_cast<const void*>(&bwd_kernel<D, false, false>));
  if ((st = set_smem_attr(kfn, C::SMEM)) != RATTN_OK) return st;
  if ((st = check_launch_regs(kfn)) != RATTN_OK) return st;
  if (det && (st = launch_bwd_dq_sm100(a, ctx, false)) != RATTN_OK) return st;
  const unsigned prep_grid = static_cast<unsigned>((rows * 16 + 255) / 256);
  if (det)
    bwd_prep_kernel<D, false><<<prep_grid, 256, 0, a.stream>>>(
        static_cast<const __nv_bfloat16*>(a.o), static_cast<const __nv_bfloat16*>(a.dout), a.delta, a.dq_acc, rows);
  else
    bwd_prep_kernel<D, true><<<prep_grid, 256, 0, a.stream>>>(
        static_cast<const __nv_bfloat16*>(a.o), static_cast<const __nv_bfloat16*>(a.dout), a.delta, a.dq_acc, rows);
  if (cudaGetLastError() != cudaSuccess) return RATTN_ERR_CUDA;
  Params p;
  p.lse = a.lse;
  p.delta = a.delta;
  p.pos = a.pos;
  p.seg = a.seg;
  p.q_pos = nullptr;
  p.kv_pos = nullptr;
  p.Lq = p.Lk = 0;
  p.accumulate = 0;
  p.BH = a.BH;
  p.group = a.group;
  p.nseg = a.nseg;
  p.Lseg = static_cast<int>(a.Lseg);
  p.nq_tiles = nt;
  p.nk_tiles = nt;
  p.causal = a.causal;
  p.kv_valid = a.kv_valid;
  p.scale = a.scale;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.dk = a.dk;
  p.dv = a.dv;
  p.err = ctx.err_word;
  p.wait_ns = ctx.wait_ns;
  const unsigned g = static_cast<unsigned>(grid);
  if (det && a.seg)
    bwd_kernel<D, true, false, false><<<g, kThreads, C::SMEM, a.stream>>>(tq, tk, tv, tdo, tdq, p);
  else if (det)
    bwd_kernel<D, false, false, false><<<g, kThreads, C::SMEM, a.stream>>>(tq, tk, tv, tdo, tdq, p);
  else if (a.seg)
    bwd_kernel<D, true, false><<<g, kThreads, C::SMEM, a.stream>>>(tq, tk, tv, tdo, tdq, p);
  else
    bwd_kernel<D, false, false><<<g, kThreads, C::SMEM, a.stream>>>(tq, tk, tv, tdo, tdq, p);
  if (cudaGetLastError() != cudaSuccess) return RATTN_ERR_CUDA;
  // Deterministic mode: dQ by one CTA per query tile, in a fixed key order.
  if (det) return launch_bwd_dq_sm100(a, ctx, true);
  const long long n4 = rows * D / 4;
  dq_convert_kernel<<<grid_for(n4, 256), 256, 0, a.stream>>>(reinterpret_cast<const float4*>(a.dq_acc),
                                                            static_cast<uint2*>(a.dq), a.scale, n4);
  return cudaGetLastError() == cudaSuccess ? RATTN_OK : RATTN_ERR_CUDA;
}

template <int D>
rattn_status launch_split(const PartialBwdArgs& a, const DevCtx& ctx) {
  using C = Cfg<D>;
  if (a.Lq > INT32_MAX - BQ || a.Lk > INT32_MAX - BK) return RATTN_ERR_UNSUPPORTED;
  if (a.group < 1 || a.BH % a.group) return RATTN_ERR_INVALID_ARG;
  const int nqt = static_cast<int>((a.Lq + BQ - 1) / BQ);
  const int nkt = static_cast<int>((a.Lk + BK - 1) / BK);
  const long long grid = static_cast<long long>(a.BH / a.group) * nkt;  // one CTA per key/value tile
  if (grid == 0) return RATTN_OK;                                       // no key rows: nothing to add
  if (grid > INT32_MAX) return RATTN_ERR_UNSUPPORTED;
  if (a.Lq == 0) {  // no query rows: the shares are zero
    if (a.accumulate) return RATTN_OK;
    const size_t bytes = static_cast<size_t>(a.BH / a.group) * static_cast<size_t>(a.Lk) * D * sizeof(float);
    if (cudaMemsetAsync(a.dk, 0, bytes, a.stream) != cudaSuccess ||
        cudaMemsetAsync(a.dv, 0, bytes, a.stream) != cudaSuccess)
      return RATTN_ERR_CUDA;
    return RATTN_OK;
  }
  CUtensorMap tq, tk, tv, tdo, tdq;
  rattn_status st;
  if ((st = make_tmap_bf16(&tq, a.q, D, a.Lq, 1, a.BH, BQ)) != RATTN_OK) return st;
  if ((st = make_tmap_bf16(&tk, a.k, D, a.Lk, 1, a.BH / a.group, BK)) != RATTN_OK) return st;
  if ((st = make_tmap_bf16(&tv, a.v, D, a.Lk, 1, a.BH / a.group, BK)) != RATTN_OK) return st;
  if ((st = make_tmap_bf16(&tdo, a.dout, D, a.Lq, 1, a.BH, BQ)) != RATTN_OK) return st;
  if ((st = make_tmap_f32_acc(&tdq, a.dq_acc, D, a.Lq, 1, a.BH)) != RATTN_OK) return st;
  const void* kfn = reinterpret_cast<const void*>(&bwd_kernel<D, false, true>);
  if ((st = set_smem_attr(kfn, C::SMEM)) != RATTN_OK) return st;
  if ((st = check_launch_regs(kfn)) != RATTN_OK) return st;
  Params p;
  p.lse = a.lse;
  p.delta = a.delta;
  p.pos = nullptr;
  p.seg = nullptr;
  p.q_pos = a.q_pos;
  p.kv_pos = a.kv_pos;
  p.BH = a.BH;
  p.group = a.group;
  p.nseg = 1;
  p.Lseg = 0;
  p.nq_tiles = nqt;
  p.nk_tiles = nkt;
  p.causal = a.causal;
  p.Lq = static_cast<int>(a.Lq);
  p.Lk = static_cast<int>(a.Lk);
  p.accumulate = a.accumulate;
  p.kv_valid = a.kv_valid;
  p.scale = a.scale;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.dk = a.dk;
  p.dv = a.dv;
  p.err = ctx.err_word;
  p.wait_ns = ctx.wait_ns;
  bwd_kernel<D, false, true><<<static_cast<unsigned>(grid), kThreads, C::SMEM, a.stream>>>(tq, tk, tv, tdo, tdq, p);
  return cudaGetLastError() == cudaSuccess ? RATTN_OK : RATTN_ERR_CUDA;
}

template <int D>
rattn_status launch_prep(const void* o, const void* dout, long long rows, float* delta, float* dq_acc,
                         cudaStream_t stream) {
  const unsigned grid = static_cast<unsigned>((rows * 16 + 255) / 256);
  if (dq_acc)
    bwd_prep_kernel<D, true><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(o),
                                                      static_cast<const __nv_bfloat16*>(dout), delta, dq_acc, rows);
  else
    bwd_prep_kernel<D, false><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(o),
                                                       static_cast<const __nv_bfloat16*>(dout), delta, dq_acc, rows);
  return cudaGetLastError() == cudaSuccess ? RATTN_OK : RATTN_ERR_CUDA;
}

}  // namespace

rattn_status launch_bwd_sm100(const BwdArgs& a, const DevCtx& ctx) {
  if (a.dtype != RATTN_BF16) return RATTN_ERR_UNSUPPORTED;
  if (a.D == 128) return launch<128>(a, ctx);
  if (a.D == 64) return launch<64>(a, ctx);
  return RATTN_ERR_UNSUPPORTED;
}

rattn_status launch_partial_bwd_sm100(const PartialBwdArgs& a, const DevCtx& ctx) {
  if (a.dtype != RATTN_BF16) return RATTN_ERR_UNSUPPORTED;
  if (a.D == 128) return launch_split<128>(a, ctx);
  if (a.D == 64) return launch_split<64>(a, ctx);
  return RATTN_ERR_UNSUPPORTED;
}

rattn_status launch_bwd_prep_sm100(const void* o, const void* dout, long long rows, int D, float* delta,
                                   float* dq_acc, cudaStream_t stream) {
  if (rows == 0) return RATTN_OK;
  if (rows > (static_cast<long long>(INT_MAX) * 256 - 255) / 16) return RATTN_ERR_UNSUPPORTED;  // grid.x limit
  if (D == 128) return launch_prep<128>(o, dout, rows, delta, dq_acc, stream);
  if (D == 64) return launch_prep<64>(o, dout, rows, delta, dq_acc, stream);
  return RATTN_ERR_UNSUPPORTED;
}

}  // namespace rattn
