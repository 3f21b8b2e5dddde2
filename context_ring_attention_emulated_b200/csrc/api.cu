// api.cu -- the C ABI entry points declared in include/rattn.h: host-side
// argument validation (nothing is launched on a bad argument), dispatch to
// the kernels, the device error word and the TMA descriptor helper.
#include <atomic>
#include <mutex>
#include <set>
#include <utility>

#include "cp_map.cuh"
#include "internal.h"

namespace rattn {

// Device-side error word written by kernels whose bounded waits gave up.
__device__ int g_err_word;
__device__ unsigned int g_work[kWorkSlots * 2];  // zero at load; see DevCtx::work

namespace {

constexpr int kMaxDevices = 64;
constexpr unsigned long long kDefaultWaitNs = 4000000000ull;

std::mutex g_mu;
std::atomic<int> g_fwd_tiling{0};
std::atomic<int> g_bwd_deterministic{0};
int* g_err_ptr[kMaxDevices] = {nullptr};
unsigned long long g_wait_ns[kMaxDevices] = {0};
int g_sm_count[kMaxDevices] = {0};
// Cached like g_err_ptr: device addresses of a context that lives as long as the process.
unsigned int* g_work_ptr[kMaxDevices] = {nullptr};
std::atomic<unsigned> g_work_next{0};
std::set<std::pair<const void*, int>> g_smem_done;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int elem_size(rattn_dtype dt) { return dt == RATTN_BF16 ? 2 : (dt == RATTN_F32 ? 4 : 0); }

// Head-dimension support per dtype: bf16 runs on the tensor cores (D = 64 or
// 128); fp32 runs the exact SIMT path (D a multiple of 4, at most 128).
rattn_status check_attn_d(int D, rattn_dtype dt) {
  if (D <= 0) return RATTN_ERR_INVALID_ARG;
  if (dt == RATTN_BF16) return (D == 64 || D == 128) ? RATTN_OK : RATTN_ERR_UNSUPPORTED;
  if (dt == RATTN_F32) return (D % 4 == 0 && D <= 128) ? RATTN_OK : RATTN_ERR_UNSUPPORTED;
  return RATTN_ERR_INVALID_ARG;
}

int64_t chunks_of(int cp, rattn_layout layout) {
  if (layout == RATTN_LAYOUT_HEAD_TAIL) return 2LL * cp;
  if (layout == RATTN_LAYOUT_CONTIGUOUS || layout == RATTN_LAYOUT_STRIPED) return cp;
  return -1;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// Kernels index (batch, head) pairs with 32-bit integers.
bool bh_fits(int B, int H) { return static_cast<int64_t>(B) * H <= INT32_MAX; }

}  // namespace

rattn_status get_dev_ctx(DevCtx* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return RATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_err_word) != cudaSuccess) return RATTN_ERR_CUDA;
    g_err_ptr[dev] = static_cast<int*>(p);
  }
  if (!g_sm_count[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
      return RATTN_ERR_CUDA;
    g_sm_count[dev] = n;
  }
  if (!g_work_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_work) != cudaSuccess) return RATTN_ERR_CUDA;
    g_work_ptr[dev] = static_cast<unsigned int*>(p);
  }
  out->sm_count = g_sm_count[dev];
  out->work = g_work_ptr[dev] + 2 * (g_work_next.fetch_add(1) % kWorkSlots);
  out->err_word = g_err_ptr[dev];
  out->wait_ns = g_wait_ns[dev] ? g_wait_ns[dev] : kDefaultWaitNs;
  out->fwd_tiling = g_fwd_tiling.load();
  out->bwd_deterministic = g_bwd_deterministic.load();
  return RATTN_OK;
}

rattn_status set_smem_attr(const void* kernel, int bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  auto key = std::make_pair(kernel, dev);
  if (g_smem_done.count(key)) return RATTN_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return RATTN_ERR_CUDA;
  g_smem_done.insert(key);
  return RATTN_OK;
}

rattn_status make_tmap_bf16(CUtensorMap* map, const void* base, int D, int64_t rows, int nseg, int64_t outer,
                            int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return RATTN_ERR_CUDA;
  if (rows < 1) rows = 1;  // an empty segment is never read; the map still needs a non-zero extent
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(nseg), static_cast<cuuint64_t>(outer)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(rows) * D * 2,
                                 static_cast<cuuint64_t>(nseg) * rows * D * 2};
  const cuuint32_t box[4] = {64u, static_cast<cuuint32_t>(box_rows), 1u, 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RATTN_OK : RATTN_ERR_CUDA;
}

rattn_status make_tmap_f32_acc(CUtensorMap* map, void* base, int D, int64_t rows, int nseg, int64_t outer,
                               int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return RATTN_ERR_CUDA;
  if (rows < 1) rows = 1;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(nseg), static_cast<cuuint64_t>(outer)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 4, static_cast<cuuint64_t>(rows) * D * 4,
                                 static_cast<cuuint64_t>(nseg) * rows * D * 4};
  const cuuint32_t box[4] = {32u, static_cast<cuuint32_t>(box_rows), 1u, 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RATTN_OK : RATTN_ERR_CUDA;
}

}  // namespace rattn

using namespace rattn;

extern "C" {

const char* rattn_status_string(rattn_status s) {
  switch (s) {
    case RATTN_OK: return "RATTN_OK";
    case RATTN_ERR_INVALID_ARG: return "RATTN_ERR_INVALID_ARG";
    case RATTN_ERR_UNSUPPORTED: return "RATTN_ERR_UNSUPPORTED";
    case RATTN_ERR_CUDA: return "RATTN_ERR_CUDA";
    case RATTN_ERR_TIMEOUT: return "RATTN_ERR_TIMEOUT";
    case RATTN_ERR_BOUNDS: return "RATTN_ERR_BOUNDS";
  }
  return "RATTN_ERR_UNKNOWN";
}

int64_t cp_layout_padded_len(int64_t L, int cp_size, rattn_layout layout) {
  if (L < 0 || cp_size < 1) return -1;
  const int64_t n = chunks_of(cp_size, layout);
  if (n < 1) return -1;
  if (L > INT64_MAX - n) return -1;
  return (L + n - 1) / n * n;
}

rattn_status cp_layout_permute(const void* x, void* y, int32_t* pos, int B, int H, int64_t L, int64_t Lp, int D,
                               rattn_dtype dtype, int cp_size, rattn_layout layout, void* stream) {
  const int es = elem_size(dtype);
  if (!es || B < 1 || H < 1 || D < 1 || L < 0 || cp_size < 1 || chunks_of(cp_size, layout) < 1)
    return RATTN_ERR_INVALID_ARG;
  if (Lp != cp_layout_padded_len(L, cp_size, layout)) return RATTN_ERR_INVALID_ARG;
  if (Lp > INT32_MAX || !bh_fits(B, H)) return RATTN_ERR_UNSUPPORTED;
  if ((static_cast<int64_t>(D) * es) % 16) return RATTN_ERR_UNSUPPORTED;
  if (Lp == 0) return RATTN_OK;
  if (!x || !y || !aligned(x, 16) || !aligned(y, 16) || (pos && !aligned(pos, 4))) return RATTN_ERR_INVALID_ARG;
  return launch_permute(x, y, pos, B * H, L, Lp, D * es, cp_size, layout, static_cast<cudaStream_t>(stream));
}

rattn_status cp_layout_unpermute(const void* y, void* x, int B, int H, int64_t L, int64_t Lp, int D,
                                 rattn_dtype dtype, int cp_size, rattn_layout layout, void* stream) {
  const int es = elem_size(dtype);
  if (!es || B < 1 || H < 1 || D < 1 || L < 0 || cp_size < 1 || chunks_of(cp_size, layout) < 1)
    return RATTN_ERR_INVALID_ARG;
  if (Lp != cp_layout_padded_len(L, cp_size, layout)) return RATTN_ERR_INVALID_ARG;
  if (Lp > INT32_MAX || !bh_fits(B, H)) return RATTN_ERR_UNSUPPORTED;
  if ((static_cast<int64_t>(D) * es) % 16) return RATTN_ERR_UNSUPPORTED;
  if (L == 0) return RATTN_OK;
  if (!x || !y || !aligned(x, 16) || !aligned(y, 16)) return RATTN_ERR_INVALID_ARG;
  return launch_unpermute(y, x, B * H, L, Lp, D * es, cp_size, layout, static_cast<cudaStream_t>(stream));
}

rattn_status cp_layout_varlen_plan(const int32_t* cu_seqlens, int nseq, int cp_size, rattn_layout layout,
                                   int64_t* Tp, int32_t* src, int32_t* pos, int32_t* segid, int32_t* gkey) {
  return cp_layout_varlen_plan_aligned(cu_seqlens, nseq, cp_size, layout, 1, Tp, src, pos, segid, gkey);
}

rattn_status cp_layout_varlen_plan_aligned(const int32_t* cu_seqlens, int nseq, int cp_size, rattn_layout layout,
                                           int align, int64_t* Tp, int32_t* src, int32_t* pos, int32_t* segid,
                                           int32_t* gkey) {
  if (!cu_seqlens || nseq < 0 || cp_size < 1 || chunks_of(cp_size, layout) < 1 || !Tp || align < 1)
    return RATTN_ERR_INVALID_ARG;
  if (cu_seqlens[0] != 0) return RATTN_ERR_INVALID_ARG;
  // Rows of each sequence's share on one rank: its padded length over cp,
  // rounded up to a multiple of align.
  auto share_rows = [&](int64_t L) {
    const int64_t n = cp_layout_padded_len(L, cp_size, layout) / cp_size;
    return (n + align - 1) / align * align;
  };
  int64_t total = 0;
  for (int i = 0; i < nseq; ++i) {
    const int64_t L = static_cast<int64_t>(cu_seqlens[i + 1]) - cu_seqlens[i];
    if (L < 0) return RATTN_ERR_INVALID_ARG;
    total += share_rows(L) * cp_size;
    if (total > INT32_MAX) return RATTN_ERR_INVALID_ARG;
  }
  *Tp = total;
  if (!src && !pos && !segid && !gkey) return RATTN_OK;
  // Rank r's slice holds, for every sequence in order, the rows rank r holds
  // when that sequence alone is permuted, then (align > 1) pad rows up to the
  // aligned share; those carry positions Lp + r * e + k past every position
  // of the sequence, so that gkey keeps increasing along the slice.
  const int64_t per_rank = total / cp_size;
  int64_t seq_off = 0, rank_off = 0;  // sequence offset in the padded pack / in a rank slice
  for (int i = 0; i < nseq; ++i) {
    const int L = cu_seqlens[i + 1] - cu_seqlens[i];
    const int Lp = static_cast<int>(cp_layout_padded_len(L, cp_size, layout));
    const int n = Lp / cp_size;
    const int n_al = static_cast<int>(share_rows(L));
    const int e = n_al - n;
    const int c = cp_map_c(Lp, cp_size, layout);
    for (int r = 0; r < cp_size; ++r) {
      for (int t = 0; t < n_al; ++t) {
        const int g = t < n ? slot_to_global(r * n + t, c, cp_size, layout) : Lp + r * e + (t - n);
        const int64_t slot = r * per_rank + rank_off + t;
        if (src) src[slot] = g < L ? cu_seqlens[i] + g : -1;
        if (pos) pos[slot] = g;
        if (segid) segid[slot] = 2 * i + (g < L ? 0 : 1);
        if (gkey) gkey[slot] = static_cast<int32_t>(seq_off + g);
      }
    }
    seq_off += static_cast<int64_t>(n_al) * cp_size;
    rank_off += n_al;
  }
  return RATTN_OK;
}

// Sizes of a packed-layout gather or scatter (pointers are checked by the callers,
// which know which of them an empty side leaves unused).
static rattn_status check_gather(int B, int H, int64_t Ta, int64_t Tb, int D, rattn_dtype dtype) {
  const int es = elem_size(dtype);
  if (!es || B < 1 || H < 1 || D < 1 || Ta < 0 || Tb < 0) return RATTN_ERR_INVALID_ARG;
  if (Ta > INT32_MAX || Tb > INT32_MAX || !bh_fits(B, H)) return RATTN_ERR_UNSUPPORTED;
  const int64_t row = static_cast<int64_t>(D) * es;
  if (row % 16 || row > 4096) return RATTN_ERR_UNSUPPORTED;
  return RATTN_OK;
}

rattn_status cp_layout_gather(const void* x, void* y, const int32_t* src, int B, int H, int64_t T_in,
                              int64_t T_out, int D, rattn_dtype dtype, void* stream) {
  rattn_status st = check_gather(B, H, T_in, T_out, D, dtype);
  if (st != RATTN_OK || T_out == 0) return st;
  if (!y || !src || !aligned(y, 16) || !aligned(src, 4) || (T_in > 0 && (!x || !aligned(x, 16))))
    return RATTN_ERR_INVALID_ARG;
  return launch_gather(T_in > 0 ? x : y, y, src, B * H, T_in, T_out, D * elem_size(dtype),
                       static_cast<cudaStream_t>(stream));
}

rattn_status cp_layout_scatter(const void* y, void* x, const int32_t* src, int B, int H, int64_t T_y,
                               int64_t T_x, int D, rattn_dtype dtype, void* stream) {
  rattn_status st = check_gather(B, H, T_y, T_x, D, dtype);
  if (st != RATTN_OK || T_y == 0 || T_x == 0) return st;
  if (!x || !y || !src || !aligned(x, 16) || !aligned(y, 16) || !aligned(src, 4)) return RATTN_ERR_INVALID_ARG;
  return launch_scatter(y, x, src, B * H, T_y, T_x, D * elem_size(dtype), static_cast<cudaStream_t>(stream));
}

static rattn_status check_rope(int B, int H, int64_t L, int64_t Lp, int D, rattn_dtype dtype, int cp_size,
                               rattn_layout layout, double base, rattn_rope_style style) {
  const int es = elem_size(dtype);
  if (!es || B < 1 || H < 1 || D < 2 || L < 0 || cp_size < 1 || chunks_of(cp_size, layout) < 1)
    return RATTN_ERR_INVALID_ARG;
  if (!(base > 0.0 && base < INFINITY)) return RATTN_ERR_INVALID_ARG;
  if (style != RATTN_ROPE_HALF && style != RATTN_ROPE_INTERLEAVED) return RATTN_ERR_INVALID_ARG;
  if (Lp != cp_layout_padded_len(L, cp_size, layout)) return RATTN_ERR_INVALID_ARG;
  if (Lp > INT32_MAX || !bh_fits(B, H)) return RATTN_ERR_UNSUPPORTED;
  const int64_t row = static_cast<int64_t>(D) * es;
  if (D % 2 || row % 16 || row > 4096) return RATTN_ERR_UNSUPPORTED;
  if (style == RATTN_ROPE_HALF && (row / 2) % 16) return RATTN_ERR_UNSUPPORTED;
  return RATTN_OK;
}

rattn_status cp_layout_permute_rope(const void* x, void* y, int32_t* pos, int B, int H, int64_t L, int64_t Lp,
                                    int D, rattn_dtype dtype, int cp_size, rattn_layout layout, double rope_base,
                                    rattn_rope_style style, void* stream) {
  rattn_status st = check_rope(B, H, L, Lp, D, dtype, cp_size, layout, rope_base, style);
  if (st != RATTN_OK) return st;
  if (Lp == 0) return RATTN_OK;
  if (!x || !y || !aligned(x, 16) || !aligned(y, 16) || (pos && !aligned(pos, 4))) return RATTN_ERR_INVALID_ARG;
  return launch_permute_rope(x, y, pos, B * H, L, Lp, D, dtype, cp_size, layout, rope_base, style,
                             static_cast<cudaStream_t>(stream));
}

rattn_status cp_layout_unpermute_rope_grad(const void* dy, void* dx, int B, int H, int64_t L, int64_t Lp, int D,
                                           rattn_dtype dtype, int cp_size, rattn_layout layout, double rope_base,
                                           rattn_rope_style style, void* stream) {
  rattn_status st = check_rope(B, H, L, Lp, D, dtype, cp_size, layout, rope_base, style);
  if (st != RATTN_OK) return st;
  if (L == 0) return RATTN_OK;
  if (!dx || !dy || !aligned(dx, 16) || !aligned(dy, 16)) return RATTN_ERR_INVALID_ARG;
  return launch_unpermute_rope_grad(dy, dx, B * H, L, Lp, D, dtype, cp_size, layout, rope_base, style,
                                    static_cast<cudaStream_t>(stream));
}

rattn_status rattn_partial_fwd(const void* q, const void* k, const void* v, const int32_t* q_pos,
                               const int32_t* kv_pos, int B, int H, int64_t Lq, int64_t Lk, int D,
                               rattn_dtype dtype, float scale, int causal, int64_t kv_valid, float* o, float* lse,
                               void* stream) {
  return rattn_partial_fwd_gqa(q, k, v, q_pos, kv_pos, B, H, H, Lq, Lk, D, dtype, scale, causal, kv_valid, o, lse,
                               stream);
}

rattn_status rattn_partial_fwd_gqa(const void* q, const void* k, const void* v, const int32_t* q_pos,
                                   const int32_t* kv_pos, int B, int H, int H_kv, int64_t Lq, int64_t Lk, int D,
                                   rattn_dtype dtype, float scale, int causal, int64_t kv_valid, float* o,
                                   float* lse, void* stream) {
  if (B < 1 || H < 1 || H_kv < 1 || H % H_kv || Lq < 0 || Lk < 0 || (causal != 0 && causal != 1) ||
      !(scale > 0.f && scale < INFINITY))
    return RATTN_ERR_INVALID_ARG;
  rattn_status st = check_attn_d(D, dtype);
  if (st != RATTN_OK) return st;
  if (Lq > INT32_MAX - 256 || Lk > INT32_MAX - 256 || !bh_fits(B, H)) return RATTN_ERR_UNSUPPORTED;
  if (Lq == 0) return RATTN_OK;
  if (!q || !o || !lse || !aligned(q, 16) || !aligned(o, 16) || !aligned(lse, 4)) return RATTN_ERR_INVALID_ARG;
  if (Lk > 0 && (!k || !v || !aligned(k, 16) || !aligned(v, 16))) return RATTN_ERR_INVALID_ARG;
  if ((q_pos && !aligned(q_pos, 4)) || (kv_pos && !aligned(kv_pos, 4))) return RATTN_ERR_INVALID_ARG;
  FwdArgs a;
  a.q = q;
  a.k = Lk > 0 ? k : q;
  a.v = Lk > 0 ? v : q;
  a.q_pos = q_pos;
  a.kv_pos = kv_pos;
  a.BH = B * H;
  a.group = H / H_kv;
  a.nseg = 1;
  a.Lq_seg = Lq;
  a.Lk_seg = Lk;
  a.D = D;
  a.dtype = dtype;
  a.scale = scale;
  a.causal = causal;
  a.kv_valid = kv_valid;
  a.o = o;
  a.o_f32 = 1;
  a.lse = lse;
  a.stream = static_cast<cudaStream_t>(stream);
  if (dtype == RATTN_BF16) {
    DevCtx ctx;
    if ((st = get_dev_ctx(&ctx)) != RATTN_OK) return st;
    return launch_fwd_sm100(a, ctx);
  }
  return launch_fwd_simt(a);
}

rattn_status rattn_merge(float* o_acc, float* lse_acc, const float* o_blk, const float* lse_blk, int B, int H,
                         int64_t Lq, int D, void* stream) {
  if (B < 1 || H < 1 || Lq < 0 || D < 4 || D % 4) return RATTN_ERR_INVALID_ARG;
  if (Lq == 0) return RATTN_OK;
  if (!o_acc || !lse_acc || !o_blk || !lse_blk || !aligned(o_acc, 16) || !aligned(o_blk, 16) ||
      !aligned(lse_acc, 4) || !aligned(lse_blk, 4))
    return RATTN_ERR_INVALID_ARG;
  return launch_merge(o_acc, lse_acc, o_blk, lse_blk, static_cast<int64_t>(B) * H * Lq, D,
                      static_cast<cudaStream_t>(stream));
}

static rattn_status check_ring(const void* q, const void* k, const void* v, const int32_t* pos, int B, int H,
                               int64_t Lp, int D, rattn_dtype dtype, int cp_size, rattn_layout layout, int causal,
                               float scale) {
  if (B < 1 || H < 1 || Lp < 0 || cp_size < 1 || (causal != 0 && causal != 1) || !(scale > 0.f && scale < INFINITY))
    return RATTN_ERR_INVALID_ARG;
  const int64_t n = chunks_of(cp_size, layout);
  if (n < 1 || Lp % n) return RATTN_ERR_INVALID_ARG;
  rattn_status st = check_attn_d(D, dtype);
  if (st != RATTN_OK) return st;
  if (cp_size > 64 || !bh_fits(B, H)) return RATTN_ERR_UNSUPPORTED;
  if (Lp > INT32_MAX - 256) return RATTN_ERR_UNSUPPORTED;
  if (Lp == 0) return RATTN_OK;
  if (!q || !k || !v || !pos || !aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(pos, 4))
    return RATTN_ERR_INVALID_ARG;
  return RATTN_OK;
}

rattn_status rattn_ring_fwd(const void* q, const void* k, const void* v, const int32_t* pos, int B, int H,
                            int64_t Lp, int D, rattn_dtype dtype, int cp_size, rattn_layout layout, int causal,
                            float scale, int64_t L_valid, void* o, float* lse, void* stream) {
  return rattn_ring_fwd_gqa(q, k, v, pos, B, H, H, Lp, D, dtype, cp_size, layout, causal, scale, L_valid, o, lse,
                            stream);
}

static rattn_status ring_fwd_impl(const void* q, const void* k, const void* v, const int32_t* pos,
                                  const int32_t* seg, int B, int H, int H_kv, int64_t Lp, int D, rattn_dtype dtype,
                                  int cp_size, rattn_layout layout, int causal, float scale, int64_t L_valid, void* o,
                                  float* lse, void* stream) {
  if (H_kv < 1 || H < 1 || H % H_kv) return RATTN_ERR_INVALID_ARG;
  rattn_status st = check_ring(q, k, v, pos, B, H, Lp, D, dtype, cp_size, layout, causal, scale);
  if (st != RATTN_OK || Lp == 0) return st;
  if (!o || !lse || !aligned(o, 16) || !aligned(lse, 4)) return RATTN_ERR_INVALID_ARG;
  FwdArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.q_pos = pos;
  a.kv_pos = pos;
  a.seg = seg;
  a.BH = B * H;
  a.group = H / H_kv;
  a.nseg = cp_size;
  a.Lq_seg = Lp / cp_size;
  a.Lk_seg = Lp / cp_size;
  a.D = D;
  a.dtype = dtype;
  a.scale = scale;
  a.causal = causal;
  a.kv_valid = L_valid;
  a.o = o;
  a.o_f32 = dtype == RATTN_F32;
  a.lse = lse;
  a.stream = static_cast<cudaStream_t>(stream);
  if (dtype == RATTN_BF16) {
    DevCtx ctx;
    if ((st = get_dev_ctx(&ctx)) != RATTN_OK) return st;
    return launch_fwd_sm100(a, ctx);
  }
  return launch_fwd_simt(a);
}

rattn_status rattn_ring_fwd_gqa(const void* q, const void* k, const void* v, const int32_t* pos, int B, int H,
                                int H_kv, int64_t Lp, int D, rattn_dtype dtype, int cp_size, rattn_layout layout,
                                int causal, float scale, int64_t L_valid, void* o, float* lse, void* stream) {
  return ring_fwd_impl(q, k, v, pos, nullptr, B, H, H_kv, Lp, D, dtype, cp_size, layout, causal, scale, L_valid, o,
                       lse, stream);
}

rattn_status rattn_ring_fwd_varlen(const void* q, const void* k, const void* v, const int32_t* gkey,
                                   const int32_t* segid, int B, int H, int H_kv, int64_t Tp, int D,
                                   rattn_dtype dtype, int cp_size, int causal, float scale, void* o, float* lse,
                                   void* stream) {
  if (Tp > 0 && (!segid || !aligned(segid, 4))) return RATTN_ERR_INVALID_ARG;
  return ring_fwd_impl(q, k, v, gkey, segid, B, H, H_kv, Tp, D, dtype, cp_size, RATTN_LAYOUT_CONTIGUOUS, causal,
                       scale, INT64_MAX, o, lse, stream);
}

size_t rattn_ring_bwd_workspace_size(int B, int H, int64_t Lp, int D) {
  if (B < 1 || H < 1 || Lp < 0 || D < 1) return 0;
  const size_t rows = static_cast<size_t>(B) * H * static_cast<size_t>(Lp);
  return round256(rows * D * sizeof(float)) + round256(rows * sizeof(float));
}

rattn_status rattn_ring_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                            const float* lse, const int32_t* pos, int B, int H, int64_t Lp, int D,
                            rattn_dtype dtype, int cp_size, rattn_layout layout, int causal, float scale,
                            int64_t L_valid, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                            void* stream) {
  return rattn_ring_bwd_gqa(q, k, v, o, dout, lse, pos, B, H, H, Lp, D, dtype, cp_size, layout, causal, scale,
                            L_valid, dq, dk, dv, workspace, workspace_bytes, stream);
}

static rattn_status ring_bwd_impl(const void* q, const void* k, const void* v, const void* o, const void* dout,
                                  const float* lse, const int32_t* pos, const int32_t* seg, int B, int H, int H_kv,
                                  int64_t Lp, int D, rattn_dtype dtype, int cp_size, rattn_layout layout, int causal,
                                  float scale, int64_t L_valid, void* dq, void* dk, void* dv, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  if (H_kv < 1 || H < 1 || H % H_kv) return RATTN_ERR_INVALID_ARG;
  rattn_status st = check_ring(q, k, v, pos, B, H, Lp, D, dtype, cp_size, layout, causal, scale);
  if (st != RATTN_OK || Lp == 0) return st;
  if (!o || !dout || !lse || !dq || !dk || !dv || !workspace || !aligned(o, 16) || !aligned(dout, 16) ||
      !aligned(lse, 4) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(workspace, 256))
    return RATTN_ERR_INVALID_ARG;
  const size_t need = rattn_ring_bwd_workspace_size(B, H, Lp, D);
  if (workspace_bytes < need) return RATTN_ERR_INVALID_ARG;
  const size_t rows = static_cast<size_t>(B) * H * static_cast<size_t>(Lp);
  BwdArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.dout = dout;
  a.lse = lse;
  a.pos = pos;
  a.seg = seg;
  a.BH = B * H;
  a.group = H / H_kv;
  a.nseg = cp_size;
  a.Lseg = Lp / cp_size;
  a.D = D;
  a.dtype = dtype;
  a.scale = scale;
  a.causal = causal;
  a.kv_valid = L_valid;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.dq_acc = static_cast<float*>(workspace);
  a.delta = reinterpret_cast<float*>(static_cast<char*>(workspace) + round256(rows * D * sizeof(float)));
  a.stream = static_cast<cudaStream_t>(stream);
  if (dtype == RATTN_BF16) {
    DevCtx ctx;
    if ((st = get_dev_ctx(&ctx)) != RATTN_OK) return st;
    return launch_bwd_sm100(a, ctx);
  }
  return launch_bwd_simt(a);
}

rattn_status rattn_ring_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const void* dout,
                                const float* lse, const int32_t* pos, int B, int H, int H_kv, int64_t Lp, int D,
                                rattn_dtype dtype, int cp_size, rattn_layout layout, int causal, float scale,
                                int64_t L_valid, void* dq, void* dk, void* dv, void* workspace,
                                size_t workspace_bytes, void* stream) {
  return ring_bwd_impl(q, k, v, o, dout, lse, pos, nullptr, B, H, H_kv, Lp, D, dtype, cp_size, layout, causal, scale,
                       L_valid, dq, dk, dv, workspace, workspace_bytes, stream);
}

rattn_status rattn_ring_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dout,
                                   const float* lse, const int32_t* gkey, const int32_t* segid, int B, int H,
                                   int H_kv, int64_t Tp, int D, rattn_dtype dtype, int cp_size, int causal,
                                   float scale, void* dq, void* dk, void* dv, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  if (Tp > 0 && (!segid || !aligned(segid, 4))) return RATTN_ERR_INVALID_ARG;
  return ring_bwd_impl(q, k, v, o, dout, lse, gkey, segid, B, H, H_kv, Tp, D, dtype, cp_size,
                       RATTN_LAYOUT_CONTIGUOUS, causal, scale, INT64_MAX, dq, dk, dv, workspace, workspace_bytes,
                       stream);
}

rattn_status rattn_bwd_prep(const void* o, const void* dout, int B, int H, int64_t L, int D, rattn_dtype dtype,
                            float* delta, float* dq_acc, void* stream) {
  if (B < 1 || H < 1 || L < 0) return RATTN_ERR_INVALID_ARG;
  rattn_status st = check_attn_d(D, dtype);
  if (st != RATTN_OK) return st;
  if (dtype != RATTN_BF16 || !bh_fits(B, H) || L > INT32_MAX) return RATTN_ERR_UNSUPPORTED;
  if (L == 0) return RATTN_OK;
  if (!o || !dout || !delta || !aligned(o, 16) || !aligned(dout, 16) || !aligned(delta, 4) ||
      (dq_acc && !aligned(dq_acc, 16)))
    return RATTN_ERR_INVALID_ARG;
  return launch_bwd_prep_sm100(o, dout, static_cast<long long>(B) * H * L, D, delta, dq_acc,
                               static_cast<cudaStream_t>(stream));
}

rattn_status rattn_partial_bwd(const void* q, const void* k, const void* v, const void* dout, const float* lse,
                               const float* delta, const int32_t* q_pos, const int32_t* kv_pos, int B, int H,
                               int H_kv, int64_t Lq, int64_t Lk, int D, rattn_dtype dtype, float scale, int causal,
                               int64_t kv_valid, float* dq_acc, float* dk, float* dv, int accumulate,
                               void* stream) {
  if (B < 1 || H < 1 || H_kv < 1 || H % H_kv || Lq < 0 || Lk < 0 || (causal != 0 && causal != 1) ||
      (accumulate != 0 && accumulate != 1) || !(scale > 0.f && scale < INFINITY))
    return RATTN_ERR_INVALID_ARG;
  rattn_status st = check_attn_d(D, dtype);
  if (st != RATTN_OK) return st;
  if (dtype != RATTN_BF16) return RATTN_ERR_UNSUPPORTED;
  if (Lq > INT32_MAX - 256 || Lk > INT32_MAX - 256 || !bh_fits(B, H)) return RATTN_ERR_UNSUPPORTED;
  if (Lk == 0) return RATTN_OK;
  if (!k || !v || !kv_pos || !dk || !dv || !aligned(k, 16) || !aligned(v, 16) || !aligned(kv_pos, 4) ||
      !aligned(dk, 16) || !aligned(dv, 16))
    return RATTN_ERR_INVALID_ARG;
  if (Lq > 0 && (!q || !dout || !lse || !delta || !q_pos || !dq_acc || !aligned(q, 16) || !aligned(dout, 16) ||
                 !aligned(lse, 4) || !aligned(delta, 4) || !aligned(q_pos, 4) || !aligned(dq_acc, 16)))
    return RATTN_ERR_INVALID_ARG;
  PartialBwdArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.dout = dout;
  a.lse = lse;
  a.delta = delta;
  a.q_pos = q_pos;
  a.kv_pos = kv_pos;
  a.BH = B * H;
  a.group = H / H_kv;
  a.Lq = Lq;
  a.Lk = Lk;
  a.D = D;
  a.dtype = dtype;
  a.scale = scale;
  a.causal = causal;
  a.kv_valid = kv_valid;
  a.dq_acc = dq_acc;
  a.dk = dk;
  a.dv = dv;
  a.accumulate = accumulate;
  a.stream = static_cast<cudaStream_t>(stream);
  DevCtx ctx;
  if ((st = get_dev_ctx(&ctx)) != RATTN_OK) return st;
  return launch_partial_bwd_sm100(a, ctx);
}

rattn_status rattn_grad_fold(float* acc, const float* blk, int64_t n, void* stream) {
  if (n < 0 || n % 4) return RATTN_ERR_INVALID_ARG;
  if (n == 0) return RATTN_OK;
  if (!acc || !blk || !aligned(acc, 16) || !aligned(blk, 16)) return RATTN_ERR_INVALID_ARG;
  return launch_grad_fold(acc, blk, n, static_cast<cudaStream_t>(stream));
}

rattn_status rattn_get_device_error(int* site) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_err_word, sizeof(int)) != cudaSuccess) return RATTN_ERR_CUDA;
  if (site) *site = v;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_err_word, &zero, sizeof(int)) != cudaSuccess) return RATTN_ERR_CUDA;
    return v >= SITE_BOUNDS ? RATTN_ERR_BOUNDS : RATTN_ERR_TIMEOUT;
  }
  return RATTN_OK;
}

rattn_status rattn_set_bwd_deterministic(int on) {
  if (on != 0 && on != 1) return RATTN_ERR_INVALID_ARG;
  g_bwd_deterministic.store(on);
  return RATTN_OK;
}

rattn_status rattn_set_fwd_tiling(int mode) {
  if (mode < 0 || mode > 4) return RATTN_ERR_INVALID_ARG;
  g_fwd_tiling.store(mode);
  return RATTN_OK;
}

rattn_status rattn_set_wait_limit_ns(unsigned long long ns) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return RATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  g_wait_ns[dev] = ns;  // 0 restores the default
  return RATTN_OK;
}

}  // extern "C"
