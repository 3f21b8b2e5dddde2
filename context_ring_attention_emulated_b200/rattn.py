"""Python binding of librattn.so (the C ABI in include/rattn.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels. Torch supplies device memory and the current stream. The library
must be built (``python -m context_ring_attention_emulated_b200.build``);
importing this module without it raises, and nothing here falls back to a CPU
or PyTorch implementation.

Functions keep the C names. Each takes tensors and infers B, H, L, D from
their shapes; outputs are allocated with torch when not supplied.
"""
import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# RATTN_DEBUG=1 selects the debug build (device-side bounds checks; built by
# ``python -m context_ring_attention_emulated_b200.build --debug``).
DEBUG = os.environ.get("RATTN_DEBUG", "0") == "1"
LIB_PATH = os.path.join(_PKG, "librattn_debug.so" if DEBUG else "librattn.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_BOUNDS = 0, 1, 2, 3, 4, 5
F32, BF16 = 0, 1
LAYOUT_CONTIGUOUS, LAYOUT_HEAD_TAIL, LAYOUT_STRIPED = 0, 1, 2
ROPE_HALF, ROPE_INTERLEAVED = 0, 1

# (name, restype, argtypes) of every symbol include/rattn.h declares.
_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_F = ctypes.c_float
_D = ctypes.c_double
SIGNATURES = [
    ("rattn_status_string", ctypes.c_char_p, [_I]),
    ("cp_layout_padded_len", _I64, [_I64, _I, _I]),
    ("cp_layout_permute", _I, [_P, _P, _P, _I, _I, _I64, _I64, _I, _I, _I, _I, _P]),
    ("cp_layout_unpermute", _I, [_P, _P, _I, _I, _I64, _I64, _I, _I, _I, _I, _P]),
    ("cp_layout_varlen_plan", _I, [_P, _I, _I, _I, ctypes.POINTER(_I64), _P, _P, _P, _P]),
    ("cp_layout_varlen_plan_aligned", _I, [_P, _I, _I, _I, _I, ctypes.POINTER(_I64), _P, _P, _P, _P]),
    ("cp_layout_gather", _I, [_P, _P, _P, _I, _I, _I64, _I64, _I, _I, _P]),
    ("cp_layout_scatter", _I, [_P, _P, _P, _I, _I, _I64, _I64, _I, _I, _P]),
    ("rattn_ring_fwd_varlen", _I, [_P, _P, _P, _P, _P, _I, _I, _I, _I64, _I, _I, _I, _I, _F, _P, _P, _P]),
    ("rattn_ring_bwd_varlen", _I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I64, _I, _I, _I, _I, _F,
                                   _P, _P, _P, _P, ctypes.c_size_t, _P]),
    ("cp_layout_permute_rope", _I, [_P, _P, _P, _I, _I, _I64, _I64, _I, _I, _I, _I, _D, _I, _P]),
    ("cp_layout_unpermute_rope_grad", _I, [_P, _P, _I, _I, _I64, _I64, _I, _I, _I, _I, _D, _I, _P]),
    ("rattn_partial_fwd", _I, [_P, _P, _P, _P, _P, _I, _I, _I64, _I64, _I, _I, _F, _I, _I64, _P, _P, _P]),
    ("rattn_partial_fwd_gqa", _I, [_P, _P, _P, _P, _P, _I, _I, _I, _I64, _I64, _I, _I, _F, _I, _I64, _P, _P,
                                   _P]),
    ("rattn_merge", _I, [_P, _P, _P, _P, _I, _I, _I64, _I, _P]),
    ("rattn_ring_fwd", _I, [_P, _P, _P, _P, _I, _I, _I64, _I, _I, _I, _I, _I, _F, _I64, _P, _P, _P]),
    ("rattn_ring_bwd_workspace_size", ctypes.c_size_t, [_I, _I, _I64, _I]),
    ("rattn_ring_bwd", _I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I64, _I, _I, _I, _I, _I, _F, _I64,
                            _P, _P, _P, _P, ctypes.c_size_t, _P]),
    ("rattn_ring_fwd_gqa", _I, [_P, _P, _P, _P, _I, _I, _I, _I64, _I, _I, _I, _I, _I, _F, _I64, _P, _P, _P]),
    ("rattn_ring_bwd_gqa", _I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I64, _I, _I, _I, _I, _I, _F, _I64,
                                _P, _P, _P, _P, ctypes.c_size_t, _P]),
    ("rattn_ring_bwd_noalloc", _I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I64, _I, _I, _I, _I, _I, _F, _I64,
                                    _P, _P, _P, _P]),
    ("rattn_bwd_prep", _I, [_P, _P, _I, _I, _I64, _I, _I, _P, _P, _P]),
    ("rattn_partial_bwd", _I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I64, _I64, _I, _I, _F, _I, _I64,
                               _P, _P, _P, _I, _P]),
    ("rattn_grad_fold", _I, [_P, _P, _I64, _P]),
    ("rattn_get_device_error", _I, [ctypes.POINTER(_I)]),
    ("rattn_set_fwd_tiling", _I, [_I]),
    ("rattn_set_bwd_deterministic", _I, [_I]),
    ("rattn_set_wait_limit_ns", _I, [ctypes.c_ulonglong]),
]


class RattnError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} failed: {status_string(code)} ({code})")
        self.code = code


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m context_ring_attention_emulated_b200.build"
                          f"{' --debug' if DEBUG else ''}` (no fallback exists)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, res, args in SIGNATURES:
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


def status_string(code):
    return lib.rattn_status_string(int(code)).decode()


def _check(fn, code):
    if code != OK:
        raise RattnError(fn, code)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def _dims(t, n, name):
    if t.dim() != n:
        raise ValueError(f"{name} must be {n}-D, got shape {tuple(t.shape)}")


def _expect(t, shape, dtype, name):
    """The library reads and writes whole [B, H, L, D] extents it cannot see:
    every tensor handed to it must have exactly the shape and dtype the call
    implies (checked here, before any launch)."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _padded(L, cp_size, layout, fn):
    Lp = cp_layout_padded_len(L, cp_size, layout)
    if Lp < 0:
        raise RattnError(fn, ERR_INVALID_ARG)
    return Lp


def _attn(q, k, v, fn, gqa=True, same_len=True):
    """Shapes of an attention call: q [B,H,Lq,D]; k, v [B,H_kv,Lk,D] in q's
    dtype; H_kv == H unless the call takes grouped heads, Lk == Lq for the
    ring calls (one sequence). Returns B, H, Lq, D, H_kv, Lk."""
    _dims(q, 4, "q")
    _dims(k, 4, "k")
    B, H, Lq, D = q.shape
    H_kv, Lk = k.shape[1], k.shape[2]
    if not gqa and H_kv != H:
        raise ValueError(f"{fn}: k and v must have the {H} heads of q, got {H_kv} (grouped heads: the _gqa call)")
    if same_len and Lk != Lq:
        raise ValueError(f"{fn}: k and v must have the {Lq} rows of q, got {Lk}")
    _expect(k, (B, H_kv, Lk, D), q.dtype, "k")
    _expect(v, (B, H_kv, Lk, D), q.dtype, "v")
    return B, H, Lq, D, H_kv, Lk


def _bwd_io(q, k, o, dout, lse, dq, dk, dv):
    B, H, L, D = q.shape
    _expect(o, q.shape, q.dtype, "o")
    _expect(dout, q.shape, q.dtype, "dout")
    _expect(lse, (B, H, L), torch.float32, "lse")
    _expect(dq, q.shape, q.dtype, "dq")
    _expect(dk, k.shape, q.dtype, "dk")
    _expect(dv, k.shape, q.dtype, "dv")


def cp_layout_padded_len(L, cp_size, layout=LAYOUT_HEAD_TAIL):
    return int(lib.cp_layout_padded_len(int(L), int(cp_size), int(layout)))


def cp_layout_permute(x, cp_size, layout=LAYOUT_HEAD_TAIL, y=None, pos=None, stream=None):
    """x [B,H,L,D] -> (y [B,H,Lp,D] rank-major, pos int32 [Lp])."""
    _dims(x, 4, "x")
    B, H, L, D = x.shape
    Lp = _padded(L, cp_size, layout, "cp_layout_permute")
    _expect(y, (B, H, Lp, D), x.dtype, "y")
    _expect(pos, (Lp,), torch.int32, "pos")
    _need_cuda(x)
    if y is None:
        y = torch.empty(B, H, Lp, D, dtype=x.dtype, device=x.device)
    if pos is None:
        pos = torch.empty(Lp, dtype=torch.int32, device=x.device)
    _need_cuda(y, pos)
    _check("cp_layout_permute", lib.cp_layout_permute(_ptr(x), _ptr(y), _ptr(pos), B, H, L, Lp, D,
                                                       _dtype_code(x), cp_size, layout, _stream(stream)))
    return y, pos


def cp_layout_unpermute(y, L, cp_size, layout=LAYOUT_HEAD_TAIL, x=None, stream=None):
    """y [B,H,Lp,D] rank-major -> x [B,H,L,D] global order."""
    _dims(y, 4, "y")
    B, H, Lp, D = y.shape
    _expect(x, (B, H, L, D), y.dtype, "x")
    _need_cuda(y)
    if x is None:
        x = torch.empty(B, H, L, D, dtype=y.dtype, device=y.device)
    _need_cuda(x)
    _check("cp_layout_unpermute", lib.cp_layout_unpermute(_ptr(y), _ptr(x), B, H, L, Lp, D, _dtype_code(y),
                                                           cp_size, layout, _stream(stream)))
    return x


def cp_layout_permute_rope(x, cp_size, layout=LAYOUT_HEAD_TAIL, rope_base=10000.0, style=ROPE_HALF, y=None,
                           pos=None, stream=None):
    """x [B,H,L,D] -> (y [B,H,Lp,D] rank-major with RoPE at the global
    positions, pos int32 [Lp])."""
    _dims(x, 4, "x")
    B, H, L, D = x.shape
    Lp = _padded(L, cp_size, layout, "cp_layout_permute_rope")
    _expect(y, (B, H, Lp, D), x.dtype, "y")
    _expect(pos, (Lp,), torch.int32, "pos")
    _need_cuda(x)
    if y is None:
        y = torch.empty(B, H, Lp, D, dtype=x.dtype, device=x.device)
    if pos is None:
        pos = torch.empty(Lp, dtype=torch.int32, device=x.device)
    _need_cuda(y, pos)
    _check("cp_layout_permute_rope", lib.cp_layout_permute_rope(
        _ptr(x), _ptr(y), _ptr(pos), B, H, L, Lp, D, _dtype_code(x), cp_size, layout, float(rope_base),
        int(style), _stream(stream)))
    return y, pos


def cp_layout_unpermute_rope_grad(dy, L, cp_size, layout=LAYOUT_HEAD_TAIL, rope_base=10000.0, style=ROPE_HALF,
                                  dx=None, stream=None):
    """dy [B,H,Lp,D] rank-major (gradient w.r.t. the rotated tensor) ->
    dx [B,H,L,D] global order (gradient w.r.t. the un-rotated input)."""
    _dims(dy, 4, "dy")
    B, H, Lp, D = dy.shape
    _expect(dx, (B, H, L, D), dy.dtype, "dx")
    _need_cuda(dy)
    if dx is None:
        dx = torch.empty(B, H, L, D, dtype=dy.dtype, device=dy.device)
    _need_cuda(dx)
    _check("cp_layout_unpermute_rope_grad", lib.cp_layout_unpermute_rope_grad(
        _ptr(dy), _ptr(dx), B, H, L, Lp, D, _dtype_code(dy), cp_size, layout, float(rope_base), int(style),
        _stream(stream)))
    return dx


def cp_layout_varlen_plan(cu_seqlens, cp_size, layout=LAYOUT_HEAD_TAIL, align=1):
    """Host-side layout of a pack of sequences (boundaries cu_seqlens, a list or
    1-D int tensor starting at 0), every sequence's share of every rank slice
    padded to a multiple of ``align`` rows (1: the plain packed layout; 128:
    no kernel tile straddles two sequences). Returns a dict of CPU int32
    tensors src, pos, segid, gkey [Tp] and Tp."""
    cu = torch.as_tensor(cu_seqlens, dtype=torch.int32).contiguous().cpu()
    nseq = cu.numel() - 1
    tp = ctypes.c_int64(0)
    fn = "cp_layout_varlen_plan_aligned"
    _check(fn, lib.cp_layout_varlen_plan_aligned(_ptr(cu), nseq, cp_size, layout, int(align), ctypes.byref(tp),
                                                 None, None, None, None))
    out = {n: torch.empty(tp.value, dtype=torch.int32) for n in ("src", "pos", "segid", "gkey")}
    _check(fn, lib.cp_layout_varlen_plan_aligned(
        _ptr(cu), nseq, cp_size, layout, int(align), ctypes.byref(tp), _ptr(out["src"]), _ptr(out["pos"]),
        _ptr(out["segid"]), _ptr(out["gkey"])))
    out["Tp"] = tp.value
    return out


def cp_layout_gather(x, src, y=None, stream=None):
    """y[:, :, i] = x[:, :, src[i]] (zero rows where src[i] < 0); src device int32."""
    _dims(x, 4, "x")
    _dims(src, 1, "src")
    B, H, T, D = x.shape
    T_out = src.numel()
    _expect(src, (T_out,), torch.int32, "src")
    _expect(y, (B, H, T_out, D), x.dtype, "y")
    _need_cuda(x, src)
    if y is None:
        y = torch.empty(B, H, T_out, D, dtype=x.dtype, device=x.device)
    _need_cuda(y)
    _check("cp_layout_gather", lib.cp_layout_gather(_ptr(x), _ptr(y), _ptr(src), B, H, T, T_out, D, _dtype_code(x),
                                                     _stream(stream)))
    return y


def cp_layout_scatter(y, src, T_x, x=None, stream=None):
    """x[:, :, src[i]] = y[:, :, i] for src[i] >= 0; x [B, H, T_x, D]."""
    _dims(y, 4, "y")
    B, H, T_y, D = y.shape
    _expect(src, (T_y,), torch.int32, "src")
    _expect(x, (B, H, T_x, D), y.dtype, "x")
    _need_cuda(y, src)
    if x is None:
        x = torch.zeros(B, H, T_x, D, dtype=y.dtype, device=y.device)
    _need_cuda(x)
    _check("cp_layout_scatter", lib.cp_layout_scatter(_ptr(y), _ptr(x), _ptr(src), B, H, T_y, T_x, D,
                                                       _dtype_code(y), _stream(stream)))
    return x


def rattn_ring_fwd_varlen(q, k, v, gkey, segid, cp_size, causal=True, scale=None, o=None, lse=None, stream=None):
    """Ring forward over a packed layout (cp_layout_varlen_plan order); gkey and
    segid device int32 [Tp]. Returns (O, LSE)."""
    B, H, Tp, D, H_kv, _ = _attn(q, k, v, "rattn_ring_fwd_varlen")
    _expect(gkey, (Tp,), torch.int32, "gkey")
    _expect(segid, (Tp,), torch.int32, "segid")
    _expect(o, q.shape, q.dtype, "o")
    _expect(lse, (B, H, Tp), torch.float32, "lse")
    _need_cuda(q, k, v, gkey, segid, o, lse)
    scale = D ** -0.5 if scale is None else scale
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty(B, H, Tp, dtype=torch.float32, device=q.device) if lse is None else lse
    _check("rattn_ring_fwd_varlen", lib.rattn_ring_fwd_varlen(
        _ptr(q), _ptr(k), _ptr(v), _ptr(gkey), _ptr(segid), B, H, H_kv, Tp, D, _dtype_code(q), cp_size, int(causal),
        float(scale), _ptr(o), _ptr(lse), _stream(stream)))
    return o, lse


def rattn_ring_bwd_varlen(q, k, v, o, dout, lse, gkey, segid, cp_size, causal=True, scale=None, dq=None, dk=None,
                          dv=None, workspace=None, stream=None):
    """Gradients of rattn_ring_fwd_varlen: returns (dQ, dK, dV)."""
    B, H, Tp, D, H_kv, _ = _attn(q, k, v, "rattn_ring_bwd_varlen")
    _expect(gkey, (Tp,), torch.int32, "gkey")
    _expect(segid, (Tp,), torch.int32, "segid")
    _bwd_io(q, k, o, dout, lse, dq, dk, dv)
    _need_cuda(q, k, v, o, dout, lse, gkey, segid, dq, dk, dv, workspace)
    scale = D ** -0.5 if scale is None else scale
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = rattn_ring_bwd_workspace_size(B, H, Tp, D)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _check("rattn_ring_bwd_varlen", lib.rattn_ring_bwd_varlen(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(gkey), _ptr(segid), B, H, H_kv, Tp, D,
        _dtype_code(q), cp_size, int(causal), float(scale), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return dq, dk, dv


def rattn_partial_fwd(q, k, v, q_pos=None, kv_pos=None, scale=None, causal=True, kv_valid=2**62,
                      o=None, lse=None, stream=None):
    """One partial attention: returns (O fp32 [B,H,Lq,D], LSE fp32 [B,H,Lq])."""
    B, H, Lq, D, _, Lk = _attn(q, k, v, "rattn_partial_fwd", gqa=False, same_len=False)
    _expect(q_pos, (Lq,), torch.int32, "q_pos")
    _expect(kv_pos, (Lk,), torch.int32, "kv_pos")
    _expect(o, (B, H, Lq, D), torch.float32, "o")
    _expect(lse, (B, H, Lq), torch.float32, "lse")
    _need_cuda(q, k, v, q_pos, kv_pos, o, lse)
    scale = D ** -0.5 if scale is None else scale
    if o is None:
        o = torch.empty(B, H, Lq, D, dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty(B, H, Lq, dtype=torch.float32, device=q.device)
    _check("rattn_partial_fwd", lib.rattn_partial_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(q_pos), _ptr(kv_pos), B, H,
                                                       Lq, Lk, D, _dtype_code(q), float(scale), int(causal),
                                                       int(kv_valid), _ptr(o), _ptr(lse), _stream(stream)))
    return o, lse


def rattn_partial_fwd_gqa(q, k, v, q_pos=None, kv_pos=None, scale=None, causal=True, kv_valid=2**62,
                          o=None, lse=None, stream=None):
    """rattn_partial_fwd with k, v [B,H_kv,Lk,D] shared by groups of H / H_kv
    query heads: returns (O fp32 [B,H,Lq,D], LSE fp32 [B,H,Lq])."""
    B, H, Lq, D, H_kv, Lk = _attn(q, k, v, "rattn_partial_fwd_gqa", same_len=False)
    _expect(q_pos, (Lq,), torch.int32, "q_pos")
    _expect(kv_pos, (Lk,), torch.int32, "kv_pos")
    _expect(o, (B, H, Lq, D), torch.float32, "o")
    _expect(lse, (B, H, Lq), torch.float32, "lse")
    _need_cuda(q, k, v, q_pos, kv_pos, o, lse)
    scale = D ** -0.5 if scale is None else scale
    if o is None:
        o = torch.empty(B, H, Lq, D, dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty(B, H, Lq, dtype=torch.float32, device=q.device)
    _check("rattn_partial_fwd_gqa", lib.rattn_partial_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(q_pos), _ptr(kv_pos),
                                                               B, H, H_kv, Lq, Lk, D, _dtype_code(q), float(scale),
                                                               int(causal), int(kv_valid), _ptr(o), _ptr(lse),
                                                               _stream(stream)))
    return o, lse


def rattn_merge(o_acc, lse_acc, o_blk, lse_blk, stream=None):
    """In-place online-softmax fold of (o_blk, lse_blk) into (o_acc, lse_acc)."""
    _dims(o_acc, 4, "o_acc")
    B, H, Lq, D = o_acc.shape
    _expect(o_acc, (B, H, Lq, D), torch.float32, "o_acc")
    _expect(o_blk, (B, H, Lq, D), torch.float32, "o_blk")
    _expect(lse_acc, (B, H, Lq), torch.float32, "lse_acc")
    _expect(lse_blk, (B, H, Lq), torch.float32, "lse_blk")
    _need_cuda(o_acc, lse_acc, o_blk, lse_blk)
    _check("rattn_merge", lib.rattn_merge(_ptr(o_acc), _ptr(lse_acc), _ptr(o_blk), _ptr(lse_blk), B, H, Lq, D,
                                           _stream(stream)))
    return o_acc, lse_acc


def rattn_ring_fwd(q, k, v, pos, cp_size, layout=LAYOUT_HEAD_TAIL, causal=True, scale=None, L_valid=None,
                   o=None, lse=None, stream=None):
    """Emulated ring forward on rank-major q/k/v [B,H,Lp,D]: returns (O, LSE)."""
    B, H, Lp, D, _, _ = _attn(q, k, v, "rattn_ring_fwd", gqa=False)
    _expect(pos, (Lp,), torch.int32, "pos")
    _expect(o, q.shape, q.dtype, "o")
    _expect(lse, (B, H, Lp), torch.float32, "lse")
    _need_cuda(q, k, v, pos, o, lse)
    scale = D ** -0.5 if scale is None else scale
    L_valid = Lp if L_valid is None else L_valid
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, H, Lp, dtype=torch.float32, device=q.device)
    _check("rattn_ring_fwd", lib.rattn_ring_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(pos), B, H, Lp, D, _dtype_code(q),
                                                 cp_size, layout, int(causal), float(scale), int(L_valid), _ptr(o),
                                                 _ptr(lse), _stream(stream)))
    return o, lse


def rattn_ring_bwd_workspace_size(B, H, Lp, D):
    return int(lib.rattn_ring_bwd_workspace_size(B, H, Lp, D))


def rattn_ring_bwd(q, k, v, o, dout, lse, pos, cp_size, layout=LAYOUT_HEAD_TAIL, causal=True, scale=None,
                   L_valid=None, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Gradients of the ring forward (rank-major): returns (dQ, dK, dV)."""
    B, H, Lp, D, _, _ = _attn(q, k, v, "rattn_ring_bwd", gqa=False)
    _expect(pos, (Lp,), torch.int32, "pos")
    _bwd_io(q, k, o, dout, lse, dq, dk, dv)
    _need_cuda(q, k, v, o, dout, lse, pos, dq, dk, dv, workspace)
    scale = D ** -0.5 if scale is None else scale
    L_valid = Lp if L_valid is None else L_valid
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = rattn_ring_bwd_workspace_size(B, H, Lp, D)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _check("rattn_ring_bwd", lib.rattn_ring_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                                                 _ptr(pos), B, H, Lp, D, _dtype_code(q), cp_size, layout,
                                                 int(causal), float(scale), int(L_valid), _ptr(dq), _ptr(dk),
                                                 _ptr(dv), _ptr(workspace), workspace.numel(), _stream(stream)))
    return dq, dk, dv


def rattn_bwd_prep(o, dout, dq_acc=True, delta=None, stream=None):
    """Delta fp32 [B,H,L] = rowsum(dout * o) for the hop-by-hop backward, and
    the zeroed fp32 dQ accumulator [B,H,L,D]. dq_acc: True allocates one,
    a tensor is zeroed in place, None skips it. Returns (delta, dq_acc)."""
    _dims(o, 4, "o")
    B, H, L, D = o.shape
    _expect(dout, o.shape, o.dtype, "dout")
    if dq_acc is not True:
        _expect(dq_acc, (B, H, L, D), torch.float32, "dq_acc")
    _expect(delta, (B, H, L), torch.float32, "delta")
    _need_cuda(o, dout)
    if dq_acc is True:
        dq_acc = torch.empty(B, H, L, D, dtype=torch.float32, device=o.device)
    if delta is None:
        delta = torch.empty(B, H, L, dtype=torch.float32, device=o.device)
    _need_cuda(dq_acc, delta)
    _check("rattn_bwd_prep", lib.rattn_bwd_prep(_ptr(o), _ptr(dout), B, H, L, D, _dtype_code(o), _ptr(delta),
                                                 _ptr(dq_acc), _stream(stream)))
    return delta, dq_acc


def rattn_partial_bwd(q, k, v, dout, lse, delta, q_pos, kv_pos, dq_acc, scale=None, causal=True, kv_valid=2**62,
                      dk=None, dv=None, accumulate=False, stream=None):
    """One hop of the backward: adds this K/V block's dQ share to dq_acc (fp32
    [B,H,Lq,D]) and returns its dK, dV shares (fp32 [B,H_kv,Lk,D]), written
    into dk / dv when given (added to them with accumulate=True)."""
    B, H, Lq, D, H_kv, Lk = _attn(q, k, v, "rattn_partial_bwd", same_len=False)
    _expect(dout, q.shape, q.dtype, "dout")
    for t, name, shape in ((lse, "lse", (B, H, Lq)), (delta, "delta", (B, H, Lq)), (q_pos, "q_pos", (Lq,)),
                           (kv_pos, "kv_pos", (Lk,)), (dq_acc, "dq_acc", (B, H, Lq, D))):
        if t is None:
            raise ValueError(f"rattn_partial_bwd: {name} is required")
        _expect(t, shape, torch.int32 if name.endswith("pos") else torch.float32, name)
    _expect(dk, (B, H_kv, Lk, D), torch.float32, "dk")
    _expect(dv, (B, H_kv, Lk, D), torch.float32, "dv")
    _need_cuda(q, k, v, dout, lse, delta, q_pos, kv_pos, dq_acc, dk, dv)
    scale = D ** -0.5 if scale is None else scale
    if accumulate and (dk is None or dv is None):
        raise ValueError("accumulate=True needs dk and dv to add to")
    dk = torch.empty(B, H_kv, Lk, D, dtype=torch.float32, device=q.device) if dk is None else dk
    dv = torch.empty(B, H_kv, Lk, D, dtype=torch.float32, device=q.device) if dv is None else dv
    _check("rattn_partial_bwd", lib.rattn_partial_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(lse),
                                                       _ptr(delta), _ptr(q_pos), _ptr(kv_pos), B, H, H_kv, Lq, Lk,
                                                       D, _dtype_code(q), float(scale), int(causal), int(kv_valid),
                                                       _ptr(dq_acc), _ptr(dk), _ptr(dv), int(bool(accumulate)),
                                                       _stream(stream)))
    return dk, dv


def rattn_grad_fold(acc, blk, stream=None):
    """acc += blk (fp32, same shape), in place; returns acc."""
    if acc.shape != blk.shape or acc.dtype != torch.float32 or blk.dtype != torch.float32:
        raise ValueError("acc and blk must be fp32 tensors of one shape")
    _need_cuda(acc, blk)
    _check("rattn_grad_fold", lib.rattn_grad_fold(_ptr(acc), _ptr(blk), acc.numel(), _stream(stream)))
    return acc


def rattn_ring_fwd_gqa(q, k, v, pos, cp_size, layout=LAYOUT_HEAD_TAIL, causal=True, scale=None, L_valid=None,
                       o=None, lse=None, stream=None):
    """Ring forward with grouped key/value heads: q [B,H,Lp,D], k/v
    [B,H_kv,Lp,D] (H_kv from k's shape); returns (O [B,H,Lp,D], LSE)."""
    B, H, Lp, D, H_kv, _ = _attn(q, k, v, "rattn_ring_fwd_gqa")
    _expect(pos, (Lp,), torch.int32, "pos")
    _expect(o, q.shape, q.dtype, "o")
    _expect(lse, (B, H, Lp), torch.float32, "lse")
    _need_cuda(q, k, v, pos, o, lse)
    scale = D ** -0.5 if scale is None else scale
    L_valid = Lp if L_valid is None else L_valid
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, H, Lp, dtype=torch.float32, device=q.device)
    _check("rattn_ring_fwd_gqa", lib.rattn_ring_fwd_gqa(
        _ptr(q), _ptr(k), _ptr(v), _ptr(pos), B, H, H_kv, Lp, D, _dtype_code(q), cp_size, layout, int(causal),
        float(scale), int(L_valid), _ptr(o), _ptr(lse), _stream(stream)))
    return o, lse


def rattn_ring_bwd_gqa(q, k, v, o, dout, lse, pos, cp_size, layout=LAYOUT_HEAD_TAIL, causal=True, scale=None,
                       L_valid=None, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Gradients of rattn_ring_fwd_gqa: returns (dQ [B,H,Lp,D], dK, dV
    [B,H_kv,Lp,D], each summed over its group of query heads)."""
    B, H, Lp, D, H_kv, _ = _attn(q, k, v, "rattn_ring_bwd_gqa")
    _expect(pos, (Lp,), torch.int32, "pos")
    _bwd_io(q, k, o, dout, lse, dq, dk, dv)
    _need_cuda(q, k, v, o, dout, lse, pos, dq, dk, dv, workspace)
    scale = D ** -0.5 if scale is None else scale
    L_valid = Lp if L_valid is None else L_valid
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = rattn_ring_bwd_workspace_size(B, H, Lp, D)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _check("rattn_ring_bwd_gqa", lib.rattn_ring_bwd_gqa(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(pos), B, H, H_kv, Lp, D, _dtype_code(q),
        cp_size, layout, int(causal), float(scale), int(L_valid), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return dq, dk, dv


def rattn_ring_bwd_noalloc(q, k, v, o, dout, lse, pos, cp_size, layout=LAYOUT_HEAD_TAIL, causal=True, scale=None,
                           L_valid=None, dq=None, dk=None, dv=None, stream=None):
    """rattn_ring_bwd without a workspace: scratch comes from the library's own
    fixed device array (for callers that cannot allocate device memory)."""
    B, H, Lp, D, _, _ = _attn(q, k, v, "rattn_ring_bwd_noalloc", gqa=False)
    _expect(pos, (Lp,), torch.int32, "pos")
    _bwd_io(q, k, o, dout, lse, dq, dk, dv)
    _need_cuda(q, k, v, o, dout, lse, pos, dq, dk, dv)
    scale = D ** -0.5 if scale is None else scale
    L_valid = Lp if L_valid is None else L_valid
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _check("rattn_ring_bwd_noalloc", lib.rattn_ring_bwd_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(pos), B, H, Lp, D, _dtype_code(q), cp_size,
        layout, int(causal), float(scale), int(L_valid), _ptr(dq), _ptr(dk), _ptr(dv), _stream(stream)))
    return dq, dk, dv


def rattn_get_device_error():
    site = ctypes.c_int(0)
    code = lib.rattn_get_device_error(ctypes.byref(site))
    return code, site.value


def rattn_set_bwd_deterministic(on):
    """True: the ring backward's dQ by a query-stationary pass (bitwise reproducible gradients)."""
    _check("rattn_set_bwd_deterministic", lib.rattn_set_bwd_deterministic(int(bool(on))))


def rattn_set_fwd_tiling(mode):
    """0: automatic, 1: one query tile per CTA, 2: two, 3: persistent (one tile per work item),
    4: 256-key tiles (D = 128)."""
    _check("rattn_set_fwd_tiling", lib.rattn_set_fwd_tiling(int(mode)))


def rattn_set_wait_limit_ns(ns):
    _check("rattn_set_wait_limit_ns", lib.rattn_set_wait_limit_ns(int(ns)))


# ------------------------------------------------------------- convenience

def ring_attention(q, k, v, cp_size, layout=LAYOUT_HEAD_TAIL, causal=True, scale=None, stream=None):
    """Global-order q/k/v [B,H,L,D] -> (O [B,H,L,D] global order, LSE fp32
    [B,H,Lp] rank-major, pos int32 [Lp]): permute to the CP layout, run the
    emulated ring, unpermute O."""
    L = q.shape[2]
    qp, pos = cp_layout_permute(q, cp_size, layout, stream=stream)
    kp, _ = cp_layout_permute(k, cp_size, layout, stream=stream)
    vp, _ = cp_layout_permute(v, cp_size, layout, stream=stream)
    o, lse = rattn_ring_fwd(qp, kp, vp, pos, cp_size, layout, causal, scale, L_valid=L, stream=stream)
    return cp_layout_unpermute(o, L, cp_size, layout, stream=stream), lse, pos
