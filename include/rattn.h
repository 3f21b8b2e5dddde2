/*
 * rattn.h -- C ABI of the B200 (sm_100a) ring-attention library with
 * context-parallel (CP) ranks emulated on one GPU.
 *
 * Sources, cited by page title and section:
 *   [CP-glossary]  Ultralytics glossary "Context Parallelism", section
 *                  "How context parallelism works" (ring attention: each device
 *                  computes a partial attention on the KV block it holds, passes
 *                  the block to the next device and repeats until the whole
 *                  sequence has been seen; exact up to ordinary rounding) and
 *                  "Practical use and trade-offs" (the 2-rank causal SDPA example
 *                  with sequence dimension 2 and a backward pass).
 *   [Megatron-CP]  Blog "Context Parallelism v.s. Sequence Parallelism
 *                  (Megatron-LM)", section "Symmetric chunk assignment" (2*cp
 *                  chunks, rank r holds chunks r and 2*cp-1-r, global position
 *                  ids follow the pairing, pad to a multiple of 2*cp).
 *   [Ring-page]    aiunderstanding.org "Sequence parallelism and ring attention",
 *                  sections "Deep dive" and "Technical insight" (local Q fixed,
 *                  K/V blocks arrive hop by hop, online softmax with a running
 *                  max and running normaliser, transfer overlapped with math).
 *
 * Conventions shared by every call:
 *   - All tensors are dense, contiguous, row-major [B, H, L, D] (sequence on
 *     dimension 2, as in [CP-glossary]'s example), in device memory owned by
 *     the caller. The library never allocates device memory; scratch space is
 *     passed in by the caller (rattn_ring_bwd's workspace).
 *   - Data pointers must be 16-byte aligned. Position arrays are int32.
 *     B * H must fit in 32 bits and sequence lengths in 31 bits (larger
 *     requests return RATTN_ERR_UNSUPPORTED).
 *   - Every compute call is asynchronous on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream). Arguments are validated on the host first;
 *     a violation returns RATTN_ERR_INVALID_ARG or RATTN_ERR_UNSUPPORTED and
 *     launches nothing. A failed launch returns RATTN_ERR_CUDA. No C++
 *     exception crosses this boundary.
 *   - dtype RATTN_BF16 runs on the tcgen05 tensor cores (bf16 operands, fp32
 *     accumulation, D in {64, 128}); RATTN_F32 runs an exact-fp32 SIMT path
 *     (D a multiple of 4, at most 128).
 *   - Position arrays must be non-decreasing within every rank's slice (ring
 *     calls) or over the whole array (rattn_partial_fwd, rattn_partial_bwd:
 *     each of q_pos and kv_pos). The layouts produced
 *     by cp_layout_permute satisfy this; kernels use it to skip and classify
 *     tiles. A key is visible to a query iff (!causal || kv_pos <= q_pos) and
 *     kv_pos < kv_valid (L_valid in ring calls).
 *   - scale (applied to q.k before the softmax) must be finite and > 0.
 *   - LSE is the natural-log softmax normaliser log(sum_j exp(scale*q.k_j))
 *     over visible keys, fp32; a query with no visible key gets LSE = -inf and
 *     O = 0.
 *   - Device-side waits are bounded. If one gives up, the kernel records an
 *     error word and returns early; rattn_get_device_error() reports it as
 *     RATTN_ERR_TIMEOUT.
 */
#ifndef RATTN_H_
#define RATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RATTN_OK = 0,
  RATTN_ERR_INVALID_ARG = 1,   /* bad pointer, size, alignment or enum       */
  RATTN_ERR_UNSUPPORTED = 2,   /* valid request the library does not handle  */
  RATTN_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed          */
  RATTN_ERR_TIMEOUT = 4,       /* a bounded device-side wait gave up         */
  RATTN_ERR_BOUNDS = 5         /* a debug build's device-side bounds check    */
                               /* failed (librattn_debug.so only)             */
} rattn_status;

typedef enum { RATTN_F32 = 0, RATTN_BF16 = 1 } rattn_dtype;

/* [Megatron-CP]: CONTIGUOUS is the naive split (rank r holds the r-th of
 * cp_size equal pieces); HEAD_TAIL is the symmetric assignment (rank r holds
 * chunk r then chunk 2*cp_size-1-r of 2*cp_size equal chunks).
 * [Ring-page] (future of sequence parallelism: striped attention rebalances
 * the causal work): STRIPED gives token g to rank g mod cp_size, each rank
 * keeping its tokens in increasing order (the Striped Attention assignment of
 * Brandon et al., 2023). */
typedef enum {
  RATTN_LAYOUT_CONTIGUOUS = 0,
  RATTN_LAYOUT_HEAD_TAIL = 1,
  RATTN_LAYOUT_STRIPED = 2
} rattn_layout;

/* Human-readable name of a status code. Never NULL. */
const char* rattn_status_string(rattn_status s);

/* [Megatron-CP] padding rule: the smallest Lp >= L that is a multiple of
 * 2*cp_size (HEAD_TAIL) or cp_size (CONTIGUOUS, STRIPED). Returns -1 on bad arguments
 * (L < 0, cp_size < 1, unknown layout). Host only; no device work. */
int64_t cp_layout_padded_len(int64_t L, int cp_size, rattn_layout layout);

/* [Megatron-CP] layout permute: x [B,H,L,D] (global order) -> y [B,H,Lp,D]
 * in rank-major order (rank r's slice is rows [r*Lp/cp, (r+1)*Lp/cp)), pad
 * rows (global index >= L) zero-filled. If pos is non-NULL it receives the
 * global position id of every slot, int32 [Lp], shared by all (b, h); pad
 * slots carry L, L+1, ... Lp must equal cp_layout_padded_len(L, cp, layout).
 * Rows must be a multiple of 16 bytes and at most 4 KB (D * sizeof(dtype)).
 * Bit-exact copy. x and y must not overlap. */
rattn_status cp_layout_permute(const void* x, void* y, int32_t* pos,
                               int B, int H, int64_t L, int64_t Lp, int D,
                               rattn_dtype dtype, int cp_size, rattn_layout layout,
                               void* stream);

/* Inverse of cp_layout_permute: y [B,H,Lp,D] -> x [B,H,L,D]; pad rows are
 * dropped. Bit-exact copy. x and y must not overlap. */
rattn_status cp_layout_unpermute(const void* y, void* x,
                                 int B, int H, int64_t L, int64_t Lp, int D,
                                 rattn_dtype dtype, int cp_size, rattn_layout layout,
                                 void* stream);

/* Rotary position embedding pairings. [Megatron-CP] "Symmetric chunk
 * assignment" requires RoPE to use every token's global position; the
 * rotation is RoFormer's (Su et al., 2021): pair i of a head vector turns by
 * the angle p * base^(-2i/D) at position p, (a, b) -> (a cos - b sin,
 * a sin + b cos). HALF pairs (x[i], x[i + D/2]) (the "rotate half" form);
 * INTERLEAVED pairs (x[2i], x[2i+1]). */
typedef enum { RATTN_ROPE_HALF = 0, RATTN_ROPE_INTERLEAVED = 1 } rattn_rope_style;

/* cp_layout_permute with RoPE fused in: y[slot] = rotate(x[g], g) where g is
 * the slot's global position (pos[slot], which is written as in
 * cp_layout_permute when pos is non-NULL); pad rows are zero. The angle is
 * formed in fp64 and reduced modulo 2*pi there; cos/sin of the remainder and
 * the rotation run in fp32, which rounds once (RNE) to dtype. Same layout, alignment and size rules as
 * cp_layout_permute, plus: rope_base finite and > 0; D even; for HALF the
 * half row D/2 * sizeof(dtype) must be a multiple of 16 bytes (bf16: D % 16
 * == 0; fp32: D % 8 == 0), else RATTN_ERR_UNSUPPORTED. x and y must not
 * overlap. */
rattn_status cp_layout_permute_rope(const void* x, void* y, int32_t* pos,
                                    int B, int H, int64_t L, int64_t Lp, int D,
                                    rattn_dtype dtype, int cp_size, rattn_layout layout,
                                    double rope_base, rattn_rope_style style, void* stream);

/* Gradient of cp_layout_permute_rope: dx [B,H,L,D] (global order) receives
 * rotate(dy[slot(g)], -angle(g)) -- the inverse rotation, which is the
 * rotation's transpose -- for dy [B,H,Lp,D] in rank-major order (the
 * gradient with respect to the permuted, rotated tensor, e.g. the dQ or dK
 * that rattn_ring_bwd returns); pad rows are dropped. Arguments and rules as
 * cp_layout_permute_rope. */
rattn_status cp_layout_unpermute_rope_grad(const void* dy, void* dx,
                                           int B, int H, int64_t L, int64_t Lp, int D,
                                           rattn_dtype dtype, int cp_size, rattn_layout layout,
                                           double rope_base, rattn_rope_style style, void* stream);

/* Packed sequences (varlen). [Megatron-CP] "Symmetric chunk assignment":
 * packed-sequence metadata must follow the pairing structure. Each sequence of
 * the pack (boundaries cu_seqlens [nseq + 1], host, starting at 0 and
 * non-decreasing) is laid out on its own: padded to its own multiple (2 *
 * cp_size for HEAD_TAIL, cp_size otherwise) and permuted as
 * cp_layout_permute would permute it alone; rank r's slice then holds rank
 * r's share of every sequence, sequences in pack order. Host only; no device
 * work. Writes Tp (the permuted pack length, a multiple of cp_size) and, when
 * the pointers are non-NULL, per slot [Tp] (host arrays):
 *   src   index into the unpadded pack, or -1 for a pad slot;
 *   pos   position inside the sequence (what RoPE uses; pads continue it);
 *   segid 2 * (sequence index) for real tokens, 2 * (sequence index) + 1 for
 *         pads: non-decreasing along every rank slice;
 *   gkey  offset of the sequence in the padded pack + pos: increasing along
 *         every rank slice.
 * Call once with the array pointers NULL to learn Tp. Returns
 * RATTN_ERR_INVALID_ARG on bad boundaries, cp_size < 1, unknown layout or a
 * pack longer than INT32_MAX slots. */
rattn_status cp_layout_varlen_plan(const int32_t* cu_seqlens, int nseq, int cp_size, rattn_layout layout,
                                   int64_t* Tp, int32_t* src, int32_t* pos, int32_t* segid, int32_t* gkey);

/* cp_layout_varlen_plan with every sequence's share of every rank slice
 * padded further, to a multiple of `align` rows (align >= 1; 1 gives
 * cp_layout_varlen_plan's layout). The page fixes only the multiple-of-2cp
 * padding; padding more keeps the pairing and changes nothing but pad slots,
 * which every attention kernel masks. With align = 128 (the kernels' tile
 * height) no 128-row tile of a rank slice straddles two sequences, so the
 * kernels skip what lies between sequences tile by tile instead of masking
 * inside tiles. The extra pad slots of rank r's share of sequence i follow its
 * real rows, with pos = Lp_i + r * e_i + k (e_i extra slots per rank,
 * k = 0..e_i-1), src = -1, segid = 2i + 1; a sequence takes cp_size times its
 * aligned share in the padded pack, and gkey = that offset + pos still
 * increases along every rank slice. RATTN_ERR_INVALID_ARG also when
 * align < 1. */
rattn_status cp_layout_varlen_plan_aligned(const int32_t* cu_seqlens, int nseq, int cp_size, rattn_layout layout,
                                           int align, int64_t* Tp, int32_t* src, int32_t* pos, int32_t* segid,
                                           int32_t* gkey);

/* Row gather for the varlen layout: y [B,H,T_out,D] with
 * y[:, :, i] = x[:, :, src[i]] for src[i] >= 0 and zero rows where
 * src[i] < 0; src is a device int32 array [T_out] with entries < T_in
 * (cp_layout_varlen_plan's src, copied to the device). Bit-exact copy; rows
 * a multiple of 16 bytes and at most 4 KB. x and y must not overlap. */
rattn_status cp_layout_gather(const void* x, void* y, const int32_t* src, int B, int H, int64_t T_in,
                              int64_t T_out, int D, rattn_dtype dtype, void* stream);

/* Inverse of cp_layout_gather for a src whose non-negative entries are
 * distinct: x[:, :, src[i]] = y[:, :, i] for src[i] >= 0 (pad rows of y are
 * dropped; rows of x that no entry names are left untouched). y [B,H,T_y,D],
 * x [B,H,T_x,D], src device int32 [T_y]. */
rattn_status cp_layout_scatter(const void* y, void* x, const int32_t* src, int B, int H, int64_t T_y,
                               int64_t T_x, int D, rattn_dtype dtype, void* stream);

/* Ring forward over a packed (varlen) layout: q [B,H,Tp,D], k and v
 * [B,H_kv,Tp,D] (H a multiple of H_kv, as rattn_ring_fwd_gqa) in the order
 * cp_layout_varlen_plan describes, with its gkey and segid arrays (device
 * int32 [Tp]). A key is visible to a query iff both carry the same even
 * segid (same sequence, not padding) and, when causal, gkey_key <= gkey_query.
 * Outputs o [B,H,Tp,D] in `dtype` and lse fp32 [B,H,Tp]; rows of pad slots
 * have lse = -inf and o = 0. Tp must be a multiple of cp_size. */
rattn_status rattn_ring_fwd_varlen(const void* q, const void* k, const void* v, const int32_t* gkey,
                                   const int32_t* segid, int B, int H, int H_kv, int64_t Tp, int D,
                                   rattn_dtype dtype, int cp_size, int causal, float scale, void* o, float* lse,
                                   void* stream);

/* Gradients of rattn_ring_fwd_varlen: dq [B,H,Tp,D]; dk, dv [B,H_kv,Tp,D].
 * Inputs as rattn_ring_fwd_varlen plus o, dout (`dtype`) and lse; workspace as
 * rattn_ring_bwd (rattn_ring_bwd_workspace_size(B, H, Tp, D) bytes). */
rattn_status rattn_ring_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dout,
                                   const float* lse, const int32_t* gkey, const int32_t* segid, int B, int H,
                                   int H_kv, int64_t Tp, int D, rattn_dtype dtype, int cp_size, int causal,
                                   float scale, void* dq, void* dk, void* dv, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* [CP-glossary], [Ring-page]: one partial attention of local queries against
 * one K/V block. q [B,H,Lq,D], k and v [B,H,Lk,D] in `dtype`; q_pos int32
 * [Lq] and kv_pos int32 [Lk] (either may be NULL, meaning 0,1,2,...);
 * keys with kv_pos >= kv_valid are masked (pass INT64_MAX for none).
 * Outputs (fp32, caller-owned): o [B,H,Lq,D] = softmax-weighted average of
 * the visible V rows, lse [B,H,Lq]. Tiles the causal relation fully masks
 * are skipped. */
rattn_status rattn_partial_fwd(const void* q, const void* k, const void* v,
                               const int32_t* q_pos, const int32_t* kv_pos,
                               int B, int H, int64_t Lq, int64_t Lk, int D,
                               rattn_dtype dtype, float scale, int causal, int64_t kv_valid,
                               float* o, float* lse, void* stream);

/* rattn_partial_fwd with grouped key/value heads ([Megatron-CP] "CP vs SP"
 * sizes the ring's K/V traffic by the key/value heads): k and v are
 * [B,H_kv,Lk,D] with H a multiple of H_kv, and query head h reads key/value
 * head h / (H / H_kv). Otherwise as rattn_partial_fwd; H_kv == H is that
 * call. RATTN_ERR_INVALID_ARG when H_kv < 1 or H % H_kv != 0. */
rattn_status rattn_partial_fwd_gqa(const void* q, const void* k, const void* v,
                                   const int32_t* q_pos, const int32_t* kv_pos,
                                   int B, int H, int H_kv, int64_t Lq, int64_t Lk, int D,
                                   rattn_dtype dtype, float scale, int causal, int64_t kv_valid,
                                   float* o, float* lse, void* stream);

/* [Ring-page] "Technical insight": online-softmax fold of a block result into
 * an accumulator, in place, fp32:
 *   LSE' = m + log(exp(LSE_acc - m) + exp(LSE_blk - m)),  m = max(LSE_acc, LSE_blk)
 *   O'   = exp(LSE_acc - LSE') O_acc + exp(LSE_blk - LSE') O_blk
 * o_acc, o_blk [B,H,Lq,D]; lse_acc, lse_blk [B,H,Lq]. A side whose LSE is
 * -inf contributes nothing; both -inf leaves LSE = -inf, O = 0. */
rattn_status rattn_merge(float* o_acc, float* lse_acc, const float* o_blk, const float* lse_blk,
                         int B, int H, int64_t Lq, int D, void* stream);

/* [CP-glossary], [Ring-page]: the whole emulated ring forward. q, k, v
 * [B,H,Lp,D] in rank-major order (as cp_layout_permute writes them) with
 * positions pos int32 [Lp], non-decreasing within each of the cp_size slices
 * (cp_layout_permute's output is): the kernels find visible and unmasked
 * tiles by binary search over them, so unsorted positions give wrong O / LSE
 * without an error (the debug build reports them as RATTN_ERR_BOUNDS). Every emulated rank r keeps its Q slice fixed and,
 * for hops t = 0..cp_size-1, attends the K/V slice of rank s = (r - t) mod
 * cp_size (blocks move to the next rank each hop), folding each block into a
 * running max / normaliser in ring order; the next block's K/V loads overlap
 * the current block's math. Keys with pos >= L_valid (padding) are masked.
 * Outputs: o [B,H,Lp,D] in `dtype` (round-to-nearest-even for bf16), lse
 * fp32 [B,H,Lp]. Lp must be a multiple of cp_size (of 2*cp_size for
 * HEAD_TAIL); 1 <= cp_size <= 64. */
rattn_status rattn_ring_fwd(const void* q, const void* k, const void* v, const int32_t* pos,
                            int B, int H, int64_t Lp, int D, rattn_dtype dtype,
                            int cp_size, rattn_layout layout, int causal, float scale,
                            int64_t L_valid, void* o, float* lse, void* stream);

/* Bytes of scratch rattn_ring_bwd needs for these sizes (fp32 dQ accumulator
 * [B,H,Lp,D] plus the per-row dot(dO, O) vector [B,H,Lp], each 256-byte
 * aligned). Host only. Returns 0 on bad arguments. */
size_t rattn_ring_bwd_workspace_size(int B, int H, int64_t Lp, int D);

/* [CP-glossary] "Practical use and trade-offs" (`.backward()` through the CP
 * attention): gradients of the ring forward, recomputing P from the saved fp32
 * LSE. Inputs as rattn_ring_fwd (pos non-decreasing within each of the cp_size
 * slices, as there) plus o (forward output, `dtype`), dout (dL/dO, `dtype`)
 * and lse (fp32). Outputs dq, dk, dv [B,H,Lp,D] in `dtype`. The
 * caller passes `workspace` (device, 256-byte aligned, at least
 * rattn_ring_bwd_workspace_size bytes); its contents on entry are ignored and
 * on return undefined. Calls sharing a workspace must not overlap. */
rattn_status rattn_ring_bwd(const void* q, const void* k, const void* v, const void* o,
                            const void* dout, const float* lse, const int32_t* pos,
                            int B, int H, int64_t Lp, int D, rattn_dtype dtype,
                            int cp_size, rattn_layout layout, int causal, float scale,
                            int64_t L_valid, void* dq, void* dk, void* dv,
                            void* workspace, size_t workspace_bytes, void* stream);

/* [Megatron-CP] "CP vs SP": the ring moves the K/V of H_kv heads, fewer than
 * the H query heads under grouped-query attention (GQA, Ainslie et al., 2023:
 * the query heads form H_kv equal groups, each group sharing one key/value
 * head). rattn_ring_fwd with grouped key/value heads: q, o [B,H,Lp,D], lse
 * [B,H,Lp]; k, v [B,H_kv,Lp,D]; H a positive multiple of H_kv; query head h
 * attends key/value head h / (H / H_kv) (contiguous groups). H_kv == H is
 * rattn_ring_fwd. H not a multiple of H_kv returns RATTN_ERR_INVALID_ARG. */
rattn_status rattn_ring_fwd_gqa(const void* q, const void* k, const void* v, const int32_t* pos,
                                int B, int H, int H_kv, int64_t Lp, int D, rattn_dtype dtype,
                                int cp_size, rattn_layout layout, int causal, float scale,
                                int64_t L_valid, void* o, float* lse, void* stream);

/* Gradients of rattn_ring_fwd_gqa: dq [B,H,Lp,D]; dk, dv [B,H_kv,Lp,D], each
 * the sum over the group's query heads (the chain rule through the shared
 * heads). q, o, dout, lse have H heads; k, v have H_kv. The workspace is sized
 * by the query heads: rattn_ring_bwd_workspace_size(B, H, Lp, D). H_kv == H
 * is rattn_ring_bwd. */
rattn_status rattn_ring_bwd_gqa(const void* q, const void* k, const void* v, const void* o,
                                const void* dout, const float* lse, const int32_t* pos,
                                int B, int H, int H_kv, int64_t Lp, int D, rattn_dtype dtype,
                                int cp_size, rattn_layout layout, int causal, float scale,
                                int64_t L_valid, void* dq, void* dk, void* dv,
                                void* workspace, size_t workspace_bytes, void* stream);

/* --- One hop at a time: the backward when CP ranks are separate processes.
 *
 * [CP-glossary] "How context parallelism works" (each device works on the
 * K/V block it holds, then passes the block on) and [Megatron-CP] "CP vs SP"
 * (K and V travel between ranks ring-style or by an all-gather): when every
 * rank is its own process, each hop of the backward is one call on the
 * rank's queries and the block in hand, and the dK, dV shares travel back to
 * the block's owner. The pages show only `.backward()`; these calls split the
 * plain softmax-attention gradient by key block: with the row's final LSE
 * and Delta_i = sum_d dO_id O_id of the whole sequence,
 *   P = exp(scale Q K^T - LSE) (masked),  dV = P^T dO,  dP = dO V^T,
 *   dS = P o (dP - Delta),  dQ = scale dS K,  dK = scale dS^T Q,
 * and the shares summed over all blocks are the gradient. bf16 only
 * (RATTN_F32 returns RATTN_ERR_UNSUPPORTED). */

/* Per-step preparation: delta fp32 [B,H,L] = rowsum(dout o o) of the bf16
 * [B,H,L,D] forward output and its upstream gradient, and, unless dq_acc is
 * NULL, zeroing of the fp32 dQ accumulator dq_acc [B,H,L,D]. */
rattn_status rattn_bwd_prep(const void* o, const void* dout, int B, int H, int64_t L, int D,
                            rattn_dtype dtype, float* delta, float* dq_acc, void* stream);

/* One hop: the share of one K/V block in the gradient of queries that
 * attend the whole sequence. q, dout [B,H,Lq,D] and lse, delta fp32 [B,H,Lq]
 * (the rank's rows; lse as the forward returned it, delta from
 * rattn_bwd_prep); k, v [B,H_kv,Lk,D] (the block; query head h reads
 * key/value head h / (H / H_kv)); q_pos int32 [Lq], kv_pos int32 [Lk], both
 * required and non-decreasing. A key is visible iff (!causal || kv_pos <=
 * q_pos) and kv_pos < kv_valid. Outputs (fp32, caller-owned, 16-byte
 * aligned): dq_acc [B,H,Lq,D] += this block's dQ; dk, dv [B,H_kv,Lk,D] =
 * the block's dK, dV shares (summed over each group's query heads), or +=
 * them when accumulate = 1. Lk = 0 does nothing; Lq = 0 writes zero shares
 * (accumulate = 0) or nothing. */
rattn_status rattn_partial_bwd(const void* q, const void* k, const void* v, const void* dout,
                               const float* lse, const float* delta, const int32_t* q_pos,
                               const int32_t* kv_pos, int B, int H, int H_kv, int64_t Lq, int64_t Lk,
                               int D, rattn_dtype dtype, float scale, int causal, int64_t kv_valid,
                               float* dq_acc, float* dk, float* dv, int accumulate, void* stream);

/* acc[i] += blk[i] for n fp32 values (n a multiple of 4, both 16-byte
 * aligned): the running dK / dV sums of a block as it travels back to its
 * owner. */
rattn_status rattn_grad_fold(float* acc, const float* blk, int64_t n, void* stream);

/* Size of the device array rattn_ring_bwd_noalloc uses as scratch space. */
#define RATTN_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/* The pages have no counterpart of this call. It is rattn_ring_bwd for
 * callers that cannot allocate device memory: code that runs where no
 * allocator is reachable (a plugin inside a host framework that owns all of
 * the device's memory, a runtime that forbids allocation after start-up, or a
 * process with a fixed memory budget), so it cannot provide a workspace.
 * Arguments, layouts and results are those of rattn_ring_bwd, without the
 * workspace. Scratch space is a RATTN_NOALLOC_SCRATCH_BYTES device array that
 * is part of the library: every GPU that loads the library keeps it until the
 * process exits, and nothing is allocated or freed by this call. A request
 * whose rattn_ring_bwd_workspace_size exceeds that size returns
 * RATTN_ERR_UNSUPPORTED and launches nothing. The first call on a device,
 * with that device current, looks up the array's device address (once per
 * device); make that first call before any stream capture on the device. The
 * looked-up address is cached for the life of the process: it assumes the
 * device's primary context is never destroyed (after cudaDeviceReset it would
 * be stale). All calls share the one array and it keeps the previous call's contents (the
 * parts that must start at zero are cleared on the device by the call
 * itself), so calls whose execution overlaps on the GPU, on any streams,
 * race on it: order them on one stream or synchronise between them. */
rattn_status rattn_ring_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                    const void* dout, const float* lse, const int32_t* pos,
                                    int B, int H, int64_t Lp, int D, rattn_dtype dtype,
                                    int cp_size, rattn_layout layout, int causal, float scale,
                                    int64_t L_valid, void* dq, void* dk, void* dv, void* stream);

/* Reads and clears the device-side error word of the current device
 * (synchronises the device). Returns RATTN_OK if no kernel recorded an
 * error, RATTN_ERR_TIMEOUT if a bounded wait gave up (*site, if non-NULL,
 * receives the recorded wait site, 1..99), RATTN_ERR_BOUNDS if a bounds check
 * of the debug build (librattn_debug.so, built with RATTN_DEBUG) failed (*site
 * receives 100 + the check's number), RATTN_ERR_CUDA if the read failed. The
 * word is process-wide per device and keeps the first failure; the library
 * caches its device address per device, assuming the device's primary
 * context lives as long as the process (after cudaDeviceReset the cached
 * address is stale). */
rattn_status rattn_get_device_error(int* site);

/* Tuning and test hook: how the bf16 attention forward (ring, GQA, packed and
 * partial calls) tiles its work, for launches made after the call, on every
 * device. 0 (the default) chooses: for unpacked calls with D = 128 and at
 * most 32 segments, 128 query rows per CTA against 256-key tiles (the score
 * product as N = 256 MMAs); else two 128-row query tiles per CTA sharing each
 * staged K/V tile when a query row attends at least 262,144 keys (cp_size x
 * slice length); else, for packed sequences, a persistent kernel (one CTA per
 * SM taking one-tile work items from a per-launch counter); else one 128-row
 * query tile per CTA against 128-key tiles. 1 forces one tile per CTA, 2 two,
 * 3 the persistent kernel, 4 the 256-key tiles (RATTN_ERR_UNSUPPORTED unless
 * D = 128 and at most 32 segments). Forms 1-3 give bit-identical O and LSE;
 * form 4 folds the keys in 256-key steps and so rounds differently (within the
 * bf16 tolerances of the others). Returns RATTN_ERR_INVALID_ARG for any other
 * mode. A persistent launch takes one of
 * 256 counter pairs in the library's device memory, zeroed again by its last
 * CTA; a launch captured in a CUDA graph keeps its pair, so replays of one
 * captured launch must not overlap each other, and more than 256 persistent
 * launches must not be in flight at once. */
rattn_status rattn_set_fwd_tiling(int mode);

/* Reproducibility switch for the ring backward (rattn_ring_bwd, _gqa, _varlen,
 * _noalloc), for launches made after the call, on every device. By default dQ
 * is accumulated by the key/value-stationary kernel with fp32 reduce-adds from
 * many CTAs, whose order varies from run to run (dK and dV are always
 * accumulated in a fixed order). With on = 1 a second, query-stationary pass
 * recomputes dQ = scale * sum_j dS_ij k_j for each 128-row query tile in one
 * CTA, over the key tiles in ring order, and writes it: dQ, dK and dV are then
 * the same, bit for bit, on every run with the same inputs, at the cost of
 * that pass (about as long as the forward). The textbook gradient of softmax
 * attention (the pages call .backward(); [CP-glossary] "Practical use and
 * trade-offs"). Returns RATTN_ERR_INVALID_ARG unless on is 0 or 1. The per-hop
 * rattn_partial_bwd is not affected. */
rattn_status rattn_set_bwd_deterministic(int on);

/* Test hook: the per-wait time limit in nanoseconds used by subsequent
 * launches on the current device (default 4e9; 0 restores the default). A
 * tiny limit makes waits give
 * up at once; kernels then drain their in-flight copies and MMAs (with a fixed
 * limit) and return without touching memory they do not own. */
rattn_status rattn_set_wait_limit_ns(unsigned long long ns);

#ifdef __cplusplus
}
#endif

#endif /* RATTN_H_ */
