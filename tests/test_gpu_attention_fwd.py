"""GPU parity of the attention forward against the fp64 oracle.

rattn_partial_fwd (one K/V block, explicit positions, masking), hop-by-hop
composition of partial + merge in ring order, and rattn_ring_fwd on the
workloads (small ones in full, full-size ones on sampled rows), both dtypes.
"""
import numpy as np
import pytest
import torch

import oracle
from context_ring_attention_emulated_b200.workloads import WORKLOADS, make_qkv, make_tensor
from tests.gpu_common import check_lse, check_o, load_rattn, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rattn():
    return load_rattn()


def _pos(n, lo, hi, seed):
    g = np.random.default_rng(seed)
    return np.sort(g.integers(lo, hi, n)).astype(np.int32)


PARTIAL_CASES = [
    # dtype, D, Lq, Lk, causal, with_pos, kv_valid
    (torch.bfloat16, 128, 128, 128, True, False, None),
    (torch.bfloat16, 128, 200, 333, True, True, None),
    (torch.bfloat16, 64, 257, 1000, True, True, 700),
    (torch.bfloat16, 64, 1, 5, False, False, None),
    (torch.bfloat16, 128, 300, 517, False, True, 400),
    (torch.bfloat16, 128, 64, 0, True, False, None),
    (torch.bfloat16, 64, 130, 130, True, True, None),
    (torch.float32, 64, 200, 333, True, True, None),
    (torch.float32, 128, 65, 97, False, False, 50),
    (torch.float32, 36, 33, 40, True, True, None),
    # more than 1024 key tiles: the tile-range searches take three rounds
    (torch.bfloat16, 64, 256, 140000, True, True, None),
    (torch.bfloat16, 128, 200, 140000, False, True, 100000),
]


@pytest.mark.parametrize("case", PARTIAL_CASES)
def test_partial_fwd(rattn, case):
    dtype, D, Lq, Lk, causal, with_pos, kv_valid = case
    B, H = 1, 2
    q = make_tensor((B, H, Lq, D), dtype, "cuda", seed=1)
    k = make_tensor((B, H, Lk, D), dtype, "cuda", seed=2)
    v = make_tensor((B, H, Lk, D), dtype, "cuda", seed=3)
    if with_pos:
        qp = _pos(Lq, 0, Lq + Lk, 4)
        kp = _pos(Lk, 0, Lq + Lk, 5)
    else:
        qp = np.arange(Lq, dtype=np.int32)
        kp = np.arange(Lk, dtype=np.int32)
    scale = D ** -0.5
    kwargs = {}
    if kv_valid is not None:
        kwargs["kv_valid"] = kv_valid
    o, lse = rattn.rattn_partial_fwd(q, k, v,
                                     torch.from_numpy(qp).cuda() if with_pos else None,
                                     torch.from_numpy(kp).cuda() if with_pos else None,
                                     scale=scale, causal=causal, **kwargs)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention(to64(q), to64(k), to64(v), scale, causal, qp, kp, kv_valid)
    check_lse(lse.cpu().numpy(), l_ref, dtype)
    check_o(o.cpu().numpy(), o_ref, dtype)


@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_hop_by_hop_partial_plus_merge_is_the_ring(rattn, dtype, D):
    """Ring order composed from the two standalone calls: for every rank r and
    hop t, rattn_partial_fwd on (Q_r, KV_{(r-t) mod cp}) then rattn_merge."""
    B, H, L, cp = 1, 2, 1000, 4
    q, k, v = (make_tensor((B, H, L, D), dtype, "cuda", seed=s) for s in (11, 12, 13))
    qp, pos = rattn.cp_layout_permute(q, cp)
    kp, _ = rattn.cp_layout_permute(k, cp)
    vp, _ = rattn.cp_layout_permute(v, cp)
    Lp = qp.shape[2]
    n = Lp // cp
    scale = D ** -0.5
    o_all = torch.empty(B, H, Lp, D, dtype=torch.float32, device="cuda")
    l_all = torch.empty(B, H, Lp, dtype=torch.float32, device="cuda")
    for r in range(cp):
        rows = slice(r * n, (r + 1) * n)
        o_acc = torch.zeros(B, H, n, D, dtype=torch.float32, device="cuda")
        l_acc = torch.full((B, H, n), float("-inf"), dtype=torch.float32, device="cuda")
        for t in range(cp):
            s = (r - t) % cp
            keys = slice(s * n, (s + 1) * n)
            ob, lb = rattn.rattn_partial_fwd(qp[:, :, rows].contiguous(), kp[:, :, keys].contiguous(),
                                             vp[:, :, keys].contiguous(), pos[rows].contiguous(),
                                             pos[keys].contiguous(), scale=scale, causal=True, kv_valid=L)
            rattn.rattn_merge(o_acc, l_acc, ob, lb)
        o_all[:, :, rows] = o_acc
        l_all[:, :, rows] = l_acc
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention(to64(q), to64(k), to64(v), scale, True)
    o_ref_p, _ = oracle.permute(o_ref, cp, oracle.HEAD_TAIL)
    l_ref_p, _ = oracle.permute(l_ref[..., None], cp, oracle.HEAD_TAIL)
    check_o(o_all.cpu().numpy(), o_ref_p, dtype)
    check_lse(l_all.cpu().numpy(), l_ref_p[..., 0], dtype)


def _ring_full_check(rattn, q, k, v, cp, layout, causal, dtype):
    L = q.shape[2]
    D = q.shape[3]
    scale = D ** -0.5
    qp, pos = rattn.cp_layout_permute(q, cp, layout)
    kp, _ = rattn.cp_layout_permute(k, cp, layout)
    vp, _ = rattn.cp_layout_permute(v, cp, layout)
    o, lse = rattn.rattn_ring_fwd(qp, kp, vp, pos, cp, layout, causal, scale, L_valid=L)
    out = rattn.cp_layout_unpermute(o, L, cp, layout)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attention(to64(q), to64(k), to64(v), scale, causal)
    check_o(out.float().cpu().numpy(), o_ref, dtype)
    real = pos.cpu().numpy() < L
    l_ref_p, _ = oracle.permute(l_ref[..., None], cp, layout)
    check_lse(lse.cpu().numpy()[..., real], l_ref_p[..., 0][..., real], dtype)
    # the output is bf16(O) rounded once: compare with the oracle rounded the same way
    return out


@pytest.mark.parametrize("name", ["fp32_L256_cp2", "bf16_L4096_cp2"])
def test_ring_fwd_small_workloads(rattn, name):
    w = WORKLOADS[name]
    q, k, v = make_qkv(w, "cuda", seed=0)
    _ring_full_check(rattn, q, k, v, w.cp, w.layout, w.causal, w.torch_dtype)


RAGGED = [
    # dtype, D, L, cp, layout, causal, B, H
    (torch.bfloat16, 128, 1000, 4, 1, True, 1, 2),     # c = 125: tiles straddle chunks, ragged last tile
    (torch.bfloat16, 64, 29, 4, 1, True, 2, 1),        # padded to 32
    (torch.bfloat16, 128, 777, 1, 1, True, 1, 1),      # one rank
    (torch.bfloat16, 128, 1000, 3, 0, False, 1, 2),    # contiguous, non-causal, 2 pad keys masked
    (torch.bfloat16, 64, 4100, 3, 1, True, 1, 1),      # padded, several tiles per hop
    (torch.bfloat16, 128, 2048, 8, 1, False, 1, 1),    # head-tail non-causal
    (torch.float32, 64, 29, 3, 1, True, 1, 2),
    (torch.float32, 128, 300, 2, 0, False, 1, 1),
    (torch.bfloat16, 128, 1000, 4, 2, True, 1, 2),     # striped: a masked diagonal tile every hop
    (torch.bfloat16, 64, 29, 4, 2, True, 2, 1),        # striped, padded to 32
    (torch.bfloat16, 128, 2048, 8, 2, False, 1, 1),    # striped non-causal
    (torch.bfloat16, 64, 4100, 3, 2, True, 1, 1),      # striped, padded, several tiles per hop
    (torch.float32, 64, 29, 3, 2, True, 1, 2),
    (torch.bfloat16, 128, 1000, 64, 1, True, 1, 2),   # the most ranks a call takes: 64 hops, 8-token chunks
    (torch.bfloat16, 64, 3000, 64, 2, True, 1, 1),    # striped, 64 ranks
    (torch.float32, 64, 500, 64, 1, True, 1, 1),      # fp32 path, 64 ranks
]


@pytest.mark.parametrize("case", RAGGED)
def test_ring_fwd_ragged_and_padded(rattn, case):
    dtype, D, L, cp, layout, causal, B, H = case
    q, k, v = (make_tensor((B, H, L, D), dtype, "cuda", seed=s) for s in (21, 22, 23))
    _ring_full_check(rattn, q, k, v, cp, layout, causal, dtype)


def _sampled_rows(L, c, n_random, seed):
    rows = set()
    for k0 in range(0, L, c):
        rows.update(range(k0, min(k0 + 4, L)))
        rows.update(range(max(k0 + c - 4, 0), min(k0 + c, L)))
    g = np.random.default_rng(seed)
    rows.update(g.integers(0, L, n_random).tolist())
    return np.array(sorted(rows))


@pytest.mark.parametrize("name,heads", [("bf16_L32000_cp4", None), ("bf16_L131072_cp8_noncausal", [0, 7]),
                                        ("bf16_L1M_cp8", [0, 5]), ("bf16_L32000_cp4_striped", [0, 31])])
def test_ring_fwd_full_size_sampled(rattn, name, heads):
    """Full-size workloads in the launch configuration the bench times;
    the oracle evaluates sampled query rows (first/last 4 of every chunk plus
    64 seeded random rows) against all keys."""
    w = WORKLOADS[name]
    q, k, v = make_qkv(w, "cuda", seed=0)
    qp, pos = rattn.cp_layout_permute(q, w.cp, w.layout)
    kp, _ = rattn.cp_layout_permute(k, w.cp, w.layout)
    vp, _ = rattn.cp_layout_permute(v, w.cp, w.layout)
    o, lse = rattn.rattn_ring_fwd(qp, kp, vp, pos, w.cp, w.layout, w.causal, w.scale, L_valid=w.L)
    torch.cuda.synchronize()
    del qp, kp, vp
    nchunk = 2 * w.cp if w.layout == 1 else w.cp
    rows = _sampled_rows(w.L, w.L // nchunk, 64, 0)
    Lp, src, pos_ref = oracle.perm_index(w.L, w.cp, w.layout)
    assert np.array_equal(pos.cpu().numpy(), pos_ref)
    slot_of = np.argsort(pos_ref)
    slots = torch.from_numpy(slot_of[rows]).cuda()
    heads = range(w.H) if heads is None else heads
    for h in heads:
        qh = to64(q[0, h, torch.from_numpy(rows).cuda()])
        kh, vh = to64(k[0, h]), to64(v[0, h])
        o_ref, l_ref = oracle.attention(qh, kh, vh, w.scale, w.causal, q_pos=rows, kv_pos=np.arange(w.L),
                                        row_block=64)
        check_o(o[0, h, slots].float().cpu().numpy(), o_ref, w.torch_dtype)
        check_lse(lse[0, h, slots].cpu().numpy(), l_ref, w.torch_dtype)
