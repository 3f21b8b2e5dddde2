"""GPU parity of packed sequences (varlen) following the layout: the library's
gather / scatter against the oracle's packed permutation (bit-exact), and the
ring forward / backward over a packed layout against the oracle's attention of
every sequence on its own (the pack is block-diagonal attention)."""
import numpy as np
import pytest
import torch

import oracle
from context_ring_attention_emulated_b200.workloads import make_tensor
from tests.gpu_common import check_grad, check_lse, check_o, load_rattn, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rattn():
    return load_rattn()


def _bits(t):
    return t.view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32).cpu().numpy()


@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128), (torch.float32, 64)])
@pytest.mark.parametrize("layout", [0, 1, 2])
@pytest.mark.parametrize("cu,cp", [([0, 5, 16, 16, 23], 2), ([0, 300, 301, 1000], 4), ([0, 64], 1)])
@pytest.mark.parametrize("align", [1, 128])
def test_gather_scatter_bit_exact(rattn, dtype, D, layout, cu, cp, align):
    T = cu[-1]
    x = make_tensor((2, 3, T, D), dtype, "cuda", seed=T + cp)
    plan = rattn.cp_layout_varlen_plan(cu, cp, layout, align)
    src = plan["src"].cuda()
    y = rattn.cp_layout_gather(x, src)
    y_ref = oracle.varlen_permute(_bits(x), cu, cp, layout, align)
    assert np.array_equal(_bits(y), y_ref)
    back = rattn.cp_layout_scatter(y, src, T)
    assert np.array_equal(_bits(back), _bits(x))


def _run(rattn, q, k, v, do, cu, cp, layout, causal, align=1):
    T = cu[-1]
    plan = rattn.cp_layout_varlen_plan(cu, cp, layout, align)
    src, gkey, segid = (plan[n].cuda() for n in ("src", "gkey", "segid"))
    qp, kp, vp, dop = (rattn.cp_layout_gather(t, src) for t in (q, k, v, do))
    scale = q.shape[-1] ** -0.5
    o, lse = rattn.rattn_ring_fwd_varlen(qp, kp, vp, gkey, segid, cp, causal, scale)
    dq, dk, dv = rattn.rattn_ring_bwd_varlen(qp, kp, vp, o, dop, lse, gkey, segid, cp, causal, scale)
    outs = [rattn.cp_layout_scatter(t, src, T) for t in (o, dq, dk, dv)]
    torch.cuda.synchronize()
    src_np = plan["src"].numpy()
    lse_g = np.full(lse.shape[:2] + (T,), np.nan)
    lse_g[..., src_np[src_np >= 0]] = lse.cpu().numpy()[..., src_np >= 0]
    # pad slots: nothing visible
    pad = src_np < 0
    if pad.any():
        assert np.all(np.isneginf(lse.cpu().numpy()[..., pad]))
    return outs, lse_g


CASES = [
    # dtype, D, cu_seqlens, cp, layout, causal, H, H_kv
    (torch.bfloat16, 128, [0, 5, 300, 300, 301, 1000], 2, 1, True, 2, 2),    # empty and 1-token sequences
    (torch.bfloat16, 128, [0, 1000, 1130, 2100], 4, 1, True, 4, 2),         # GQA, sequences spanning tiles
    (torch.bfloat16, 64, [0, 77, 500, 520, 900], 3, 2, True, 2, 1),         # striped, MQA
    (torch.bfloat16, 128, [0, 200, 700, 701], 2, 0, False, 2, 2),           # contiguous, non-causal
    (torch.bfloat16, 128, [0, 4000, 4001, 5000], 4, 1, False, 1, 1),        # head-tail non-causal
    (torch.float32, 64, [0, 5, 40, 41, 100], 2, 1, True, 2, 2),
    (torch.float32, 32, [0, 30, 90], 3, 2, False, 2, 1),
]


@pytest.mark.parametrize("align", [1, 128])
@pytest.mark.parametrize("case", CASES)
def test_ring_varlen_fwd_bwd_per_sequence(rattn, case, align):
    dtype, D, cu, cp, layout, causal, H, H_kv = case
    T = cu[-1]
    q = make_tensor((1, H, T, D), dtype, "cuda", seed=81)
    k, v = (make_tensor((1, H_kv, T, D), dtype, "cuda", seed=s) for s in (82, 83))
    do = make_tensor((1, H, T, D), dtype, "cuda", seed=84)
    (o, dq, dk, dv), lse = _run(rattn, q, k, v, do, cu, cp, layout, causal, align)
    scale = D ** -0.5
    for i in range(len(cu) - 1):
        a, b = cu[i], cu[i + 1]
        if a == b:
            continue
        qs, ks, vs, ds = to64(q[..., a:b, :]), to64(k[..., a:b, :]), to64(v[..., a:b, :]), to64(do[..., a:b, :])
        ke, ve = oracle.gqa_expand(ks, H), oracle.gqa_expand(vs, H)
        o_ref, l_ref = oracle.attention(qs, ke, ve, scale, causal)
        check_o(o[..., a:b, :].float().cpu().numpy(), o_ref, dtype)
        check_lse(lse[..., a:b], l_ref, dtype)
        dq_ref, dke, dve = oracle.attention_bwd(qs, ke, ve, ds, scale, causal)
        check_grad(dq[..., a:b, :].float().cpu().numpy(), dq_ref)
        check_grad(dk[..., a:b, :].float().cpu().numpy(), oracle.gqa_reduce(dke, H_kv))
        check_grad(dv[..., a:b, :].float().cpu().numpy(), oracle.gqa_reduce(dve, H_kv))


@pytest.mark.parametrize("align", [1, 128])
def test_ring_varlen_32k_pack(rattn, align):
    """A 32,000-token pack of 24 documents of mixed lengths (64 to 3000
    tokens), 8 heads, D = 128, cp = 4 head-tail, causal, in the plain and the
    tile-aligned packed layout: every sequence of heads 0 and 7 against the
    oracle, forward and backward."""
    g = np.random.default_rng(7)
    lens = g.integers(64, 3000, 23)
    lens = np.append(lens, 32000 - lens.sum()) if lens.sum() < 32000 else lens
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(int).tolist()
    cu = [c for c in cu if c <= 32000]
    if cu[-1] != 32000:
        cu.append(32000)
    H, D, cp = 8, 128, 4
    q, k, v, do = (make_tensor((1, H, 32000, D), torch.bfloat16, "cuda", seed=s) for s in (91, 92, 93, 94))
    (o, dq, dk, dv), lse = _run(rattn, q, k, v, do, cu, cp, 1, True, align)
    scale = D ** -0.5
    for h in (0, 7):
        for i in range(len(cu) - 1):
            a, b = cu[i], cu[i + 1]
            qs, ks, vs, ds = (to64(t[0, h, a:b]) for t in (q, k, v, do))
            o_ref, l_ref = oracle.attention(qs, ks, vs, scale, True)
            check_o(o[0, h, a:b].float().cpu().numpy(), o_ref, torch.bfloat16)
            check_lse(lse[0, h, a:b], l_ref, torch.bfloat16)
            grads = oracle.attention_bwd(qs, ks, vs, ds, scale, True)
            for got, ref in zip((dq, dk, dv), grads):
                check_grad(got[0, h, a:b].float().cpu().numpy(), ref)
