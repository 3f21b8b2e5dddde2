// internal.h -- host-side declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "rattn.h"

namespace rattn {

// Per-device context every launch carries: the device-side error word and the
// bounded-wait limit.
struct DevCtx {
  int* err_word;
  unsigned long long wait_ns;
  int fwd_tiling;  // 0 automatic, 1 one query tile per CTA, 2 two, 3 persistent, 4 256-key tiles (rattn_set_fwd_tiling)
  int sm_count;    // multiprocessors of the device (persistent grids)
  int bwd_deterministic;  // 1: dQ of the ring backward by the query-stationary pass (rattn_set_bwd_deterministic)
  // A pair of work counters for one persistent launch (next work item, CTAs
  // finished), zero when the launch starts; its last CTA zeroes them again.
  // Each context fetch takes the next of kWorkSlots pairs, so launches in
  // flight on different streams use different pairs.
  unsigned int* work;
};
constexpr int kWorkSlots = 256;
rattn_status get_dev_ctx(DevCtx* out);

// Wait sites recorded in the error word.
enum WaitSite : int {
  SITE_FWD_LOAD = 1,
  SITE_FWD_MMA = 2,
  SITE_FWD_SOFTMAX = 3,
  SITE_FWD_EPILOGUE = 4,
  SITE_BWD_LOAD = 5,
  SITE_BWD_MMA = 6,
  SITE_BWD_COMPUTE = 7,
  SITE_BWD_EPILOGUE = 8,
  SITE_DRAIN = 9,
  SITE_BOUNDS = 100,  // + check number: a debug build's bounds check failed
};

// 4-D bf16 tensor map over [outer][nseg][rows][D] with a (64 x box_rows) box
// and 128-byte swizzle; rows past `rows` read as zero.
rattn_status make_tmap_bf16(CUtensorMap* map, const void* base, int D, int64_t rows, int nseg, int64_t outer,
                            int box_rows);

// 4-D fp32 tensor map over [outer][nseg][rows][D] with a (32 x box_rows) box
// and 128-byte swizzle, for tile reduce-adds into an accumulator; rows past
// `rows` are outside the tensor (reduce-adds there are dropped).
rattn_status make_tmap_f32_acc(CUtensorMap* map, void* base, int D, int64_t rows, int nseg, int64_t outer,
                               int box_rows = 128);

// Sets the max dynamic shared memory attribute of a kernel once per device.
rattn_status set_smem_attr(const void* kernel, int bytes);

// Attention forward over segments: q viewed as [BH][nseg][Lq_seg][D], k/v as
// [BH][nseg][Lk_seg][D]; query segment r attends key segments (r - t) mod nseg
// for t = 0..nseg-1 (nseg = 1 for a single partial attention).
struct FwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const int32_t* q_pos;   // [nseg*Lq_seg] or NULL (row index)
  const int32_t* kv_pos;  // [nseg*Lk_seg] or NULL (row index)
  const int32_t* seg = nullptr;  // packed sequences: segid per slot (shared by q and kv), or NULL
  int BH;         // batch x query heads
  int group = 1;  // query heads per key/value head (GQA); K/V hold BH / group heads
  int nseg;
  int64_t Lq_seg;
  int64_t Lk_seg;
  int D;
  rattn_dtype dtype;
  float scale;
  int causal;
  int64_t kv_valid;
  void* o;        // [BH][nseg*Lq_seg][D]
  int o_f32;      // 1: fp32 output, 0: output in `dtype`
  float* lse;     // [BH][nseg*Lq_seg]
  cudaStream_t stream;
};
rattn_status launch_fwd_sm100(const FwdArgs& a, const DevCtx& ctx);
rattn_status launch_fwd_sm100_pair(const FwdArgs& a, const DevCtx& ctx);  // two query tiles per CTA
rattn_status launch_fwd_sm100_persist(const FwdArgs& a, const DevCtx& ctx);  // persistent, one tile per item
rattn_status launch_fwd_sm100_wide(const FwdArgs& a, const DevCtx& ctx);  // 256-key tiles (D = 128)
rattn_status launch_fwd_simt(const FwdArgs& a);

struct BwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* o;
  const void* dout;
  const float* lse;
  const int32_t* pos;  // [nseg*Lseg]
  const int32_t* seg = nullptr;  // packed sequences: segid per slot, or NULL
  int BH;              // batch x query heads
  int group = 1;       // query heads per key/value head (GQA); K/V, dK, dV hold BH / group heads
  int nseg;
  int64_t Lseg;
  int D;
  rattn_dtype dtype;
  float scale;
  int causal;
  int64_t kv_valid;
  void* dq;
  void* dk;
  void* dv;
  float* dq_acc;  // workspace [BH][nseg*Lseg][D] fp32
  float* delta;   // workspace [BH][nseg*Lseg] fp32
  cudaStream_t stream;
};
rattn_status launch_bwd_sm100(const BwdArgs& a, const DevCtx& ctx);
// The query-stationary dQ pass (attn_bwd_dq_sm100.cu): dq (bf16) from q, k, v,
// dout, lse, delta and the positions of a; run = false only prepares and
// checks everything on the host (so that a later failure cannot follow a
// launch).
rattn_status launch_bwd_dq_sm100(const BwdArgs& a, const DevCtx& ctx, bool run);

// One hop of the ring backward with query rows of one rank and key rows of
// another: q, dout [BH][Lq][D], lse, delta [BH][Lq], q_pos [Lq]; k, v
// [BH/group][Lk][D], kv_pos [Lk]. dq_acc (fp32 [BH][Lq][D]) receives
// scale * dS K added; dk, dv (fp32 [BH/group][Lk][D]) receive the block's
// shares, written (accumulate = 0) or added (1).
struct PartialBwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* dout;
  const float* lse;
  const float* delta;
  const int32_t* q_pos;
  const int32_t* kv_pos;
  int BH;
  int group;
  int64_t Lq;
  int64_t Lk;
  int D;
  rattn_dtype dtype;
  float scale;
  int causal;
  int64_t kv_valid;
  float* dq_acc;
  float* dk;
  float* dv;
  int accumulate;
  cudaStream_t stream;
};
rattn_status launch_partial_bwd_sm100(const PartialBwdArgs& a, const DevCtx& ctx);
// Delta = rowsum(dO o O) over `rows` bf16 rows of D, and zeroing of dq_acc
// (fp32, same rows) unless it is NULL.
rattn_status launch_bwd_prep_sm100(const void* o, const void* dout, long long rows, int D, float* delta,
                                   float* dq_acc, cudaStream_t stream);
rattn_status launch_bwd_simt(const BwdArgs& a);

rattn_status launch_permute(const void* x, void* y, int32_t* pos, int BH, int64_t L, int64_t Lp, int row_bytes,
                            int cp, int layout, cudaStream_t stream);
rattn_status launch_gather(const void* x, void* y, const int32_t* src, int BH, int64_t T_in, int64_t T_out,
                           int row_bytes, cudaStream_t stream);
rattn_status launch_scatter(const void* y, void* x, const int32_t* src, int BH, int64_t T_y, int64_t T_x,
                            int row_bytes, cudaStream_t stream);
rattn_status launch_unpermute(const void* y, void* x, int BH, int64_t L, int64_t Lp, int row_bytes, int cp,
                              int layout, cudaStream_t stream);
rattn_status launch_permute_rope(const void* x, void* y, int32_t* pos, int BH, int64_t L, int64_t Lp, int D,
                                 rattn_dtype dtype, int cp, int layout, double base, int style, cudaStream_t stream);
rattn_status launch_unpermute_rope_grad(const void* dy, void* dx, int BH, int64_t L, int64_t Lp, int D,
                                        rattn_dtype dtype, int cp, int layout, double base, int style,
                                        cudaStream_t stream);
rattn_status launch_grad_fold(float* acc, const float* blk, int64_t n, cudaStream_t stream);
rattn_status launch_merge(float* o_acc, float* lse_acc, const float* o_blk, const float* lse_blk, int64_t rows,
                          int D, cudaStream_t stream);

}  // namespace rattn
