"""CPU tests of the C-ABI library: it builds for sm_100a, loads, exports every
symbol include/rattn.h declares, and rejects bad arguments on the host before
any device work (no compute call runs here: this machine has no GPU)."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from tests.gpu_common import load_rattn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rattn.h")


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", src, flags=re.M)) - {"if", "defined"})


@pytest.fixture(scope="module")
def rattn():
    return load_rattn()


def test_every_declared_symbol_is_exported(rattn):
    names = header_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(rattn.lib, n), f"{n} declared in rattn.h but not exported"
    assert sorted(n for n, _, _ in rattn.SIGNATURES) == names


def test_debug_build_compiles_and_exports_every_symbol():
    """The RATTN_DEBUG variant (device-side bounds checks) builds from the same
    sources and exports the same C ABI."""
    from context_ring_attention_emulated_b200 import build as b
    path = b.build(debug=True)
    assert os.path.basename(path) == "librattn_debug.so"
    lib = ctypes.CDLL(path)
    for n in header_functions():
        assert hasattr(lib, n), f"{n} missing from the debug build"


def test_bwd_deterministic_switch_rejects_other_values(rattn):
    for on in (-1, 2, 5):
        assert rattn.lib.rattn_set_bwd_deterministic(on) == rattn.ERR_INVALID_ARG
    for on in (1, 0):
        assert rattn.lib.rattn_set_bwd_deterministic(on) == rattn.OK


def test_fwd_tiling_hook_rejects_unknown_modes(rattn):
    for mode in (-1, 5, 7):
        assert rattn.lib.rattn_set_fwd_tiling(mode) == rattn.ERR_INVALID_ARG
    for mode in (1, 2, 3, 4, 0):
        assert rattn.lib.rattn_set_fwd_tiling(mode) == rattn.OK


def test_status_strings(rattn):
    for code, name in enumerate(["RATTN_OK", "RATTN_ERR_INVALID_ARG", "RATTN_ERR_UNSUPPORTED", "RATTN_ERR_CUDA",
                                 "RATTN_ERR_TIMEOUT", "RATTN_ERR_BOUNDS"]):
        assert rattn.status_string(code) == name
    assert rattn.status_string(99) == "RATTN_ERR_UNKNOWN"


@pytest.mark.parametrize("L,cp,layout,expect", [
    (32000, 4, 1, 32000), (4096, 2, 1, 4096), (1048576, 8, 1, 1048576), (131072, 8, 0, 131072),
    (10, 4, 1, 16), (10, 4, 0, 12), (0, 3, 1, 0), (1, 1, 1, 2), (1, 1, 0, 1),
    (-1, 2, 1, -1), (10, 0, 1, -1), (10, 2, 7, -1), (10, 4, 2, 12), (32000, 4, 2, 32000), (0, 3, 2, 0)])
def test_padded_len(rattn, L, cp, layout, expect):
    assert rattn.lib.cp_layout_padded_len(L, cp, layout) == expect


def test_padded_len_matches_oracle(rattn):
    import oracle
    for cp in range(1, 17):
        for L in (0, 1, 5, 63, 64, 65, 1000):
            for layout in (0, 1, 2):
                assert rattn.lib.cp_layout_padded_len(L, cp, layout) == oracle.padded_len(L, cp, layout)


FAKE = 0x10000        # 16-byte aligned fake device address (never dereferenced)
MIS = 0x10004         # misaligned


def test_permute_rejects_bad_arguments(rattn):
    L = rattn.lib
    # Lp does not match the padding rule
    assert L.cp_layout_permute(FAKE, FAKE, FAKE, 1, 1, 10, 12, 64, 1, 4, 1, None) == rattn.ERR_INVALID_ARG
    # bad sizes / enums
    assert L.cp_layout_permute(FAKE, FAKE, FAKE, 0, 1, 16, 16, 64, 1, 4, 1, None) == rattn.ERR_INVALID_ARG
    assert L.cp_layout_permute(FAKE, FAKE, FAKE, 1, 1, 16, 16, 64, 5, 4, 1, None) == rattn.ERR_INVALID_ARG
    assert L.cp_layout_permute(FAKE, FAKE, FAKE, 1, 1, 16, 16, 64, 1, 0, 1, None) == rattn.ERR_INVALID_ARG
    # null / misaligned pointers
    assert L.cp_layout_permute(None, FAKE, FAKE, 1, 1, 16, 16, 64, 1, 4, 1, None) == rattn.ERR_INVALID_ARG
    assert L.cp_layout_permute(MIS, FAKE, FAKE, 1, 1, 16, 16, 64, 1, 4, 1, None) == rattn.ERR_INVALID_ARG
    # row not a multiple of 16 bytes
    assert L.cp_layout_permute(FAKE, FAKE, FAKE, 1, 1, 16, 16, 3, 1, 4, 1, None) == rattn.ERR_UNSUPPORTED
    # empty sequence is a no-op
    assert L.cp_layout_permute(FAKE, FAKE, FAKE, 1, 1, 0, 0, 64, 1, 4, 1, None) == rattn.OK
    assert L.cp_layout_unpermute(FAKE, FAKE, 1, 1, 10, 12, 64, 1, 4, 1, None) == rattn.ERR_INVALID_ARG
    assert L.cp_layout_unpermute(MIS, FAKE, 1, 1, 16, 16, 64, 1, 4, 1, None) == rattn.ERR_INVALID_ARG


def test_rope_permute_rejects_bad_arguments(rattn):
    L = rattn.lib
    pr = lambda **kw: L.cp_layout_permute_rope(kw.get("x", FAKE), FAKE, FAKE, 1, 1, kw.get("L", 16),
                                               kw.get("Lp", 16), kw.get("D", 64), kw.get("dt", 1), 4,
                                               kw.get("layout", 1), ctypes.c_double(kw.get("base", 1e4)),
                                               kw.get("style", 0), None)
    assert pr(base=0.0) == rattn.ERR_INVALID_ARG
    assert pr(base=float("inf")) == rattn.ERR_INVALID_ARG
    assert pr(base=float("nan")) == rattn.ERR_INVALID_ARG
    assert pr(style=2) == rattn.ERR_INVALID_ARG
    assert pr(Lp=24) == rattn.ERR_INVALID_ARG
    assert pr(layout=5) == rattn.ERR_INVALID_ARG
    assert pr(x=MIS) == rattn.ERR_INVALID_ARG
    assert pr(x=None) == rattn.ERR_INVALID_ARG
    assert pr(D=8, style=0) == rattn.ERR_UNSUPPORTED      # bf16 HALF: half row of 8 bytes
    assert pr(D=4, dt=0, style=0) == rattn.ERR_UNSUPPORTED
    assert pr(D=3, dt=0, style=1) == rattn.ERR_UNSUPPORTED
    assert pr(D=4096) == rattn.ERR_UNSUPPORTED            # row above 4 KB
    assert pr(L=0, Lp=0) == rattn.OK
    ug = lambda **kw: L.cp_layout_unpermute_rope_grad(kw.get("dy", FAKE), FAKE, 1, 1, kw.get("L", 16),
                                                      kw.get("Lp", 16), 64, 1, 4, 1,
                                                      ctypes.c_double(kw.get("base", 1e4)), kw.get("style", 1), None)
    assert ug(base=-1.0) == rattn.ERR_INVALID_ARG
    assert ug(dy=MIS) == rattn.ERR_INVALID_ARG
    assert ug(Lp=32) == rattn.ERR_INVALID_ARG
    assert ug(L=0, Lp=0) == rattn.OK


def test_gqa_calls_reject_bad_arguments(rattn):
    L = rattn.lib
    fwd = lambda H, Hkv: L.rattn_ring_fwd_gqa(FAKE, FAKE, FAKE, FAKE, 1, H, Hkv, 256, 64, 1, 2, 1, 1,
                                              ctypes.c_float(0.125), 256, FAKE, FAKE, None)
    assert fwd(4, 3) == rattn.ERR_INVALID_ARG      # H not a multiple of H_kv
    assert fwd(4, 0) == rattn.ERR_INVALID_ARG
    assert fwd(2, 4) == rattn.ERR_INVALID_ARG
    bwd = lambda H, Hkv: L.rattn_ring_bwd_gqa(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, H, Hkv, 256, 64, 1, 2, 1,
                                              1, ctypes.c_float(0.125), 256, FAKE, FAKE, FAKE, FAKE, 1 << 30, None)
    assert bwd(6, 4) == rattn.ERR_INVALID_ARG
    assert bwd(4, -2) == rattn.ERR_INVALID_ARG


def test_attention_calls_reject_bad_arguments(rattn):
    L = rattn.lib
    ring = lambda **kw: L.rattn_ring_fwd(kw.get("q", FAKE), FAKE, FAKE, kw.get("pos", FAKE), 1, 2,
                                         kw.get("Lp", 256), kw.get("D", 64), kw.get("dt", 1), kw.get("cp", 2),
                                         kw.get("layout", 1), kw.get("causal", 1), ctypes.c_float(0.125), 256,
                                         kw.get("o", FAKE), FAKE, None)
    assert ring(cp=0) == rattn.ERR_INVALID_ARG
    assert ring(Lp=250) == rattn.ERR_INVALID_ARG          # not a multiple of 2*cp
    assert ring(layout=3) == rattn.ERR_INVALID_ARG
    assert ring(causal=2) == rattn.ERR_INVALID_ARG
    assert ring(D=96) == rattn.ERR_UNSUPPORTED            # bf16 tensor-core path: D in {64, 128}
    assert ring(D=132, dt=0) == rattn.ERR_UNSUPPORTED     # fp32 path: D <= 128, multiple of 4
    assert ring(cp=65, Lp=130 * 2) == rattn.ERR_UNSUPPORTED
    assert ring(q=MIS) == rattn.ERR_INVALID_ARG
    assert ring(pos=None) == rattn.ERR_INVALID_ARG
    assert ring(o=None) == rattn.ERR_INVALID_ARG
    assert ring(Lp=0) == rattn.OK
    part = lambda **kw: L.rattn_partial_fwd(kw.get("q", FAKE), FAKE, FAKE, None, None, 1, 1, kw.get("Lq", 8), 8,
                                            kw.get("D", 64), 1, ctypes.c_float(kw.get("scale", 0.1)), 1, 1 << 40,
                                            kw.get("o", FAKE), FAKE, None)
    assert part(Lq=-1) == rattn.ERR_INVALID_ARG
    assert part(scale=float("nan")) == rattn.ERR_INVALID_ARG
    assert part(q=MIS) == rattn.ERR_INVALID_ARG
    assert part(o=MIS) == rattn.ERR_INVALID_ARG
    assert part(D=80) == rattn.ERR_UNSUPPORTED
    assert part(Lq=0) == rattn.OK
    gqa = lambda H, H_kv, Lq=8: L.rattn_partial_fwd_gqa(FAKE, FAKE, FAKE, None, None, 1, H, H_kv, Lq, 8, 64, 1,
                                                         ctypes.c_float(0.1), 1, 1 << 40, FAKE, FAKE, None)
    assert gqa(4, 3) == rattn.ERR_INVALID_ARG            # H not a multiple of H_kv
    assert gqa(4, 0) == rattn.ERR_INVALID_ARG
    assert gqa(4, 8) == rattn.ERR_INVALID_ARG
    assert gqa(8, 2, Lq=0) == rattn.OK
    assert L.rattn_merge(FAKE, FAKE, FAKE, FAKE, 1, 1, 4, 6, None) == rattn.ERR_INVALID_ARG
    assert L.rattn_merge(MIS, FAKE, FAKE, FAKE, 1, 1, 4, 8, None) == rattn.ERR_INVALID_ARG
    assert L.rattn_merge(FAKE, FAKE, FAKE, FAKE, 1, 1, 0, 8, None) == rattn.OK


def test_bwd_rejects_bad_arguments_and_sizes_workspace(rattn):
    L = rattn.lib
    need = L.rattn_ring_bwd_workspace_size(1, 32, 32000, 128)
    rows = 32 * 32000
    assert need == ((rows * 128 * 4 + 255) // 256) * 256 + ((rows * 4 + 255) // 256) * 256
    assert L.rattn_ring_bwd_workspace_size(0, 1, 1, 1) == 0

    def bwd(ws=FAKE, ws_bytes=need, **kw):
        return L.rattn_ring_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 32, 32000, 128, 1, 4, 1, 1,
                                ctypes.c_float(0.088), 32000, FAKE, FAKE, kw.get("dv", FAKE), ws, ws_bytes, None)
    assert bwd(ws_bytes=need - 1) == rattn.ERR_INVALID_ARG
    assert bwd(ws=FAKE + 16) == rattn.ERR_INVALID_ARG   # workspace must be 256-byte aligned
    assert bwd(ws=None) == rattn.ERR_INVALID_ARG
    assert bwd(dv=None) == rattn.ERR_INVALID_ARG


@pytest.mark.parametrize("layout", [0, 1, 2])
@pytest.mark.parametrize("cp", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("cu", [[0, 5, 16, 16, 23], [0, 64], [0], [0, 1, 2, 3], [0, 4000, 4001, 9000, 32000]])
@pytest.mark.parametrize("align", [1, 8, 128])
def test_varlen_plan_matches_oracle(rattn, layout, cp, cu, align):
    """The library's host-side packed layout against the oracle's, slot by slot
    (plain and aligned); the kernels' segid is 2 * sequence (+1 for padding)."""
    import oracle
    plan = rattn.cp_layout_varlen_plan(cu, cp, layout, align)
    Tp, src, pos, seg, gkey = oracle.varlen_index(cu, cp, layout, align)
    assert plan["Tp"] == Tp
    assert np.array_equal(plan["src"].numpy(), src)
    assert np.array_equal(plan["pos"].numpy(), pos)
    assert np.array_equal(plan["gkey"].numpy(), gkey)
    # every pad slot belongs to its sequence's block: recover the sequence of each slot from gkey
    sizes = [-(-oracle.padded_len(b - a, cp, layout) // cp // align) * align * cp for a, b in zip(cu, cu[1:])]
    offsets = np.cumsum([0] + sizes)
    slot_seq = np.searchsorted(offsets, gkey, side="right") - 1 if Tp else np.zeros(0, int)
    assert np.array_equal(plan["segid"].numpy(), 2 * slot_seq + (src < 0))
    assert np.array_equal(np.where(src >= 0, slot_seq, -1), seg)
    assert sum(sizes) == Tp


def test_varlen_calls_reject_bad_arguments(rattn):
    L = rattn.lib
    tp = ctypes.c_int64(0)
    bad = torch.tensor([0, 5, 3], dtype=torch.int32)
    assert L.cp_layout_varlen_plan(bad.data_ptr(), 2, 2, 1, ctypes.byref(tp), None, None, None, None) == \
        rattn.ERR_INVALID_ARG
    start = torch.tensor([1, 5], dtype=torch.int32)
    assert L.cp_layout_varlen_plan(start.data_ptr(), 1, 2, 1, ctypes.byref(tp), None, None, None, None) == \
        rattn.ERR_INVALID_ARG
    ok = torch.tensor([0, 5], dtype=torch.int32)
    assert L.cp_layout_varlen_plan(ok.data_ptr(), 1, 0, 1, ctypes.byref(tp), None, None, None, None) == \
        rattn.ERR_INVALID_ARG
    for align in (0, -128):
        assert L.cp_layout_varlen_plan_aligned(ok.data_ptr(), 1, 2, 1, align, ctypes.byref(tp), None, None, None,
                                               None) == rattn.ERR_INVALID_ARG
    assert L.cp_layout_varlen_plan_aligned(ok.data_ptr(), 1, 2, 1, 128, ctypes.byref(tp), None, None, None,
                                           None) == rattn.OK and tp.value == 256
    assert L.cp_layout_gather(FAKE, FAKE, FAKE, 1, 1, 16, 16, 3, 1, None) == rattn.ERR_UNSUPPORTED
    assert L.cp_layout_gather(FAKE, MIS, FAKE, 1, 1, 16, 16, 64, 1, None) == rattn.ERR_INVALID_ARG
    assert L.cp_layout_gather(FAKE, FAKE, FAKE, 1, 1, 16, 0, 64, 1, None) == rattn.OK
    assert L.cp_layout_scatter(FAKE, FAKE, None, 1, 1, 16, 16, 64, 1, None) == rattn.ERR_INVALID_ARG
    fv = L.rattn_ring_fwd_varlen(FAKE, FAKE, FAKE, FAKE, None, 1, 2, 2, 256, 64, 1, 2, 1, ctypes.c_float(0.125),
                                 FAKE, FAKE, None)
    assert fv == rattn.ERR_INVALID_ARG            # segid required
    fv = L.rattn_ring_fwd_varlen(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 2, 255, 64, 1, 2, 1, ctypes.c_float(0.125),
                                 FAKE, FAKE, None)
    assert fv == rattn.ERR_INVALID_ARG            # Tp not a multiple of cp


def test_batch_times_heads_beyond_int32_is_unsupported(rattn):
    L = rattn.lib
    big = 1 << 16
    assert L.cp_layout_permute(FAKE, FAKE, FAKE, big, big, 16, 16, 64, 1, 4, 1, None) == rattn.ERR_UNSUPPORTED
    assert L.cp_layout_unpermute(FAKE, FAKE, big, big, 16, 16, 64, 1, 4, 1, None) == rattn.ERR_UNSUPPORTED
    assert L.cp_layout_gather(FAKE, FAKE, FAKE, big, big, 16, 16, 64, 1, None) == rattn.ERR_UNSUPPORTED
    assert L.rattn_ring_fwd(FAKE, FAKE, FAKE, FAKE, big, big, 256, 64, 1, 2, 1, 1, ctypes.c_float(0.125), 256,
                            FAKE, FAKE, None) == rattn.ERR_UNSUPPORTED


def test_hop_backward_calls_reject_bad_arguments(rattn):
    """rattn_bwd_prep, rattn_partial_bwd and rattn_grad_fold validate on the
    host and launch nothing on a bad argument."""
    L, E, U, OK = rattn.lib, rattn.ERR_INVALID_ARG, rattn.ERR_UNSUPPORTED, rattn.OK
    BF16, F32 = rattn.BF16, rattn.F32
    # prep: sizes, dtype, pointers; an empty sequence is a no-op
    assert L.rattn_bwd_prep(FAKE, FAKE, 0, 1, 8, 64, BF16, FAKE, FAKE, None) == E
    assert L.rattn_bwd_prep(FAKE, FAKE, 1, 1, 8, 64, F32, FAKE, FAKE, None) == U
    assert L.rattn_bwd_prep(FAKE, FAKE, 1, 1, 8, 96, BF16, FAKE, FAKE, None) == U
    assert L.rattn_bwd_prep(MIS, FAKE, 1, 1, 8, 64, BF16, FAKE, FAKE, None) == E
    assert L.rattn_bwd_prep(FAKE, FAKE, 1, 1, 8, 64, BF16, None, FAKE, None) == E
    assert L.rattn_bwd_prep(FAKE, FAKE, 1, 1, 8, 64, BF16, FAKE, MIS, None) == E
    assert L.rattn_bwd_prep(FAKE, FAKE, 1, 1, 0, 64, BF16, FAKE, FAKE, None) == OK

    def hop(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, dout=FAKE, lse=FAKE, delta=FAKE, q_pos=FAKE, kv_pos=FAKE, B=1, H=4, H_kv=2,
                 Lq=256, Lk=256, D=128, dtype=BF16, scale=0.1, causal=1, kv_valid=2**62, dq=FAKE, dk=FAKE, dv=FAKE,
                 acc=0)
        a.update(kw)
        return L.rattn_partial_bwd(a["q"], a["k"], a["v"], a["dout"], a["lse"], a["delta"], a["q_pos"],
                                   a["kv_pos"], a["B"], a["H"], a["H_kv"], a["Lq"], a["Lk"], a["D"], a["dtype"],
                                   a["scale"], a["causal"], a["kv_valid"], a["dq"], a["dk"], a["dv"], a["acc"], None)
    assert hop(H_kv=3) == E                  # H not a multiple of H_kv
    assert hop(acc=2) == E and hop(causal=2) == E and hop(scale=0.0) == E and hop(Lq=-1) == E
    assert hop(dtype=F32, D=64) == U         # tensor-core path only
    assert hop(D=96) == U
    assert hop(kv_pos=None) == E and hop(q_pos=None) == E and hop(dk=MIS) == E and hop(dq=None) == E
    assert hop(k=MIS) == E and hop(lse=0x10002) == E
    assert hop(Lk=0) == OK                   # no keys: nothing to add
    assert hop(B=2**16, H=2**16, H_kv=2**16) == U
    # fold: n a multiple of 4, aligned pointers; n = 0 is a no-op
    assert L.rattn_grad_fold(FAKE, FAKE, 6, None) == E
    assert L.rattn_grad_fold(FAKE, FAKE, -4, None) == E
    assert L.rattn_grad_fold(MIS, FAKE, 8, None) == E
    assert L.rattn_grad_fold(FAKE, None, 8, None) == E
    assert L.rattn_grad_fold(FAKE, FAKE, 0, None) == OK


def test_binding_checks_shapes_and_dtypes_before_any_launch(rattn):
    """The library cannot see tensor extents: the binding refuses tensors whose
    shape or dtype does not match the call (before its CUDA check, so this runs
    here on CPU tensors), and lets matching ones through to that check."""
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    t = lambda *s, d=bf: torch.zeros(*s, dtype=d)
    q, kv, pos = t(1, 4, 16, 64), t(1, 4, 16, 64), t(16, d=i32)
    bad = [
        lambda: rattn.cp_layout_permute(q, 2, y=t(1, 4, 8, 64)),
        lambda: rattn.cp_layout_permute(q, 2, pos=t(16, d=torch.int64)),
        lambda: rattn.cp_layout_unpermute(q, 16, 2, x=t(1, 4, 16, 64, d=f32)),
        lambda: rattn.cp_layout_gather(q, t(16, d=torch.int64)),
        lambda: rattn.cp_layout_gather(q, pos, y=t(1, 4, 15, 64)),
        lambda: rattn.cp_layout_scatter(q, t(15, d=i32), 16),
        lambda: rattn.rattn_ring_fwd(q, t(1, 2, 16, 64), t(1, 2, 16, 64), pos, 2),     # grouped heads: _gqa call
        lambda: rattn.rattn_ring_fwd(q, kv, kv, t(15, d=i32), 2),
        lambda: rattn.rattn_ring_fwd(q, kv, kv, pos, 2, o=t(1, 4, 16, 64, d=f32)),
        lambda: rattn.rattn_ring_fwd(q, kv, kv, pos, 2, lse=t(1, 4, 16)),
        lambda: rattn.rattn_ring_fwd(q, kv.float(), kv, pos, 2),
        lambda: rattn.rattn_ring_bwd(q, kv, kv, q, q.float(), t(1, 4, 16, d=f32), pos, 2),
        lambda: rattn.rattn_ring_bwd(q, kv, kv, q, q, t(1, 4, 16, d=f32), pos, 2, dk=t(1, 4, 8, 64)),
        lambda: rattn.rattn_ring_fwd_gqa(q, t(1, 2, 16, 64), t(1, 4, 16, 64), pos, 2),
        lambda: rattn.rattn_ring_bwd_noalloc(q, kv, kv, q, q, t(1, 4, 15, d=f32), pos, 2),
        lambda: rattn.rattn_partial_fwd(q, t(1, 2, 9, 64), t(1, 2, 9, 64)),
        lambda: rattn.rattn_partial_fwd(q, t(1, 4, 9, 64), t(1, 4, 9, 64), q_pos=t(9, d=i32)),
        lambda: rattn.rattn_merge(t(1, 4, 16, 64, d=f32), t(1, 4, 16, d=f32), q, t(1, 4, 16, d=f32)),
        lambda: rattn.rattn_bwd_prep(q, q, dq_acc=t(1, 4, 16, 64)),
        lambda: rattn.rattn_bwd_prep(q, q, delta=t(1, 4, 15, d=f32)),
        lambda: rattn.rattn_partial_bwd(q, kv, kv, q, t(1, 4, 16, d=f32), t(1, 4, 16, d=f32), None, pos,
                                        t(1, 4, 16, 64, d=f32)),
        lambda: rattn.rattn_partial_bwd(q, kv, kv, q, t(1, 4, 16, d=f32), t(1, 4, 16, d=f32), pos, pos,
                                        t(1, 4, 16, 64, d=f32), dk=t(1, 4, 16, 64)),
        lambda: rattn.rattn_grad_fold(t(8, d=f32), t(8)),
        lambda: rattn.rattn_ring_fwd_varlen(q, kv, kv, t(15, d=i32), pos, 2),
    ]
    for i, call in enumerate(bad):
        with pytest.raises(ValueError) as e:
            call()
        assert "CUDA" not in str(e.value), f"case {i} reached the CUDA check: {e.value}"
    with pytest.raises(rattn.RattnError):
        rattn.cp_layout_permute(q, 0)                   # no padded length for cp = 0
    good = [
        lambda: rattn.cp_layout_permute(q, 2),
        lambda: rattn.rattn_ring_fwd(q, kv, kv, pos, 2),
        lambda: rattn.rattn_ring_fwd_gqa(q, t(1, 2, 16, 64), t(1, 2, 16, 64), pos, 2),
        lambda: rattn.rattn_partial_fwd(q, t(1, 4, 9, 64), t(1, 4, 9, 64), t(16, d=i32), t(9, d=i32)),
        lambda: rattn.rattn_partial_bwd(q, t(1, 2, 9, 64), t(1, 2, 9, 64), q, t(1, 4, 16, d=f32),
                                        t(1, 4, 16, d=f32), pos, t(9, d=i32), t(1, 4, 16, 64, d=f32)),
        lambda: rattn.rattn_bwd_prep(q, q),
    ]
    for call in good:
        with pytest.raises(ValueError, match="CUDA"):
            call()
