"""GPU parity of the ring forward and backward with grouped key/value heads
(GQA: H query heads share H_kv key/value heads in contiguous groups) against
the fp64 oracle on expanded heads, with dK/dV summed per group."""
import numpy as np
import pytest
import torch

import oracle
from context_ring_attention_emulated_b200.workloads import WORKLOADS, make_qkv, make_tensor
from tests.gpu_common import check_grad, check_lse, check_o, load_rattn, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rattn():
    return load_rattn()


CASES = [
    # dtype, D, L, cp, layout, causal, B, H, H_kv
    (torch.bfloat16, 128, 1000, 4, 1, True, 1, 4, 2),
    (torch.bfloat16, 64, 777, 3, 2, True, 2, 6, 1),       # MQA, striped, padded
    (torch.bfloat16, 128, 2048, 2, 0, False, 1, 8, 2),    # contiguous, non-causal
    (torch.bfloat16, 128, 29, 4, 1, True, 1, 3, 3),       # group of one through the GQA entry points
    (torch.float32, 64, 300, 2, 1, True, 1, 4, 2),
    (torch.float32, 32, 100, 4, 0, False, 2, 6, 3),
]


def _run(rattn, q, k, v, do, cp, layout, causal):
    L, D = q.shape[2], q.shape[3]
    scale = D ** -0.5
    qp, pos = rattn.cp_layout_permute(q, cp, layout)
    kp, _ = rattn.cp_layout_permute(k, cp, layout)
    vp, _ = rattn.cp_layout_permute(v, cp, layout)
    dop, _ = rattn.cp_layout_permute(do, cp, layout)
    o, lse = rattn.rattn_ring_fwd_gqa(qp, kp, vp, pos, cp, layout, causal, scale, L_valid=L)
    dq, dk, dv = rattn.rattn_ring_bwd_gqa(qp, kp, vp, o, dop, lse, pos, cp, layout, causal, scale, L_valid=L)
    outs = [rattn.cp_layout_unpermute(t, L, cp, layout) for t in (o, dq, dk, dv)]
    torch.cuda.synchronize()
    return outs, lse, pos


@pytest.mark.parametrize("case", CASES)
def test_ring_gqa_fwd_bwd(rattn, case):
    dtype, D, L, cp, layout, causal, B, H, H_kv = case
    q = make_tensor((B, H, L, D), dtype, "cuda", seed=61)
    k, v = (make_tensor((B, H_kv, L, D), dtype, "cuda", seed=s) for s in (62, 63))
    do = make_tensor((B, H, L, D), dtype, "cuda", seed=64)
    (o, dq, dk, dv), lse, pos = _run(rattn, q, k, v, do, cp, layout, causal)
    scale = D ** -0.5
    ke, ve = oracle.gqa_expand(to64(k), H), oracle.gqa_expand(to64(v), H)
    o_ref, l_ref = oracle.attention(to64(q), ke, ve, scale, causal)
    check_o(o.float().cpu().numpy(), o_ref, dtype)
    real = pos.cpu().numpy() < L
    l_ref_p, _ = oracle.permute(l_ref[..., None], cp, layout)
    check_lse(lse.cpu().numpy()[..., real], l_ref_p[..., 0][..., real], dtype)
    dq_ref, dke, dve = oracle.attention_bwd(to64(q), ke, ve, to64(do), scale, causal)
    check_grad(dq.float().cpu().numpy(), dq_ref)
    check_grad(dk.float().cpu().numpy(), oracle.gqa_reduce(dke, H_kv))
    check_grad(dv.float().cpu().numpy(), oracle.gqa_reduce(dve, H_kv))


def test_ring_gqa_matches_mha_on_repeated_heads(rattn):
    """Independent of the oracle: GQA on H_kv heads equals the MHA entry points
    on K/V repeated to H heads (the forward bit for bit: the same tiles), and
    its dK/dV equal the MHA gradients summed over each group."""
    B, H, H_kv, L, D, cp = 1, 8, 2, 4096, 128, 4
    q = make_tensor((B, H, L, D), torch.bfloat16, "cuda", seed=71)
    k, v = (make_tensor((B, H_kv, L, D), torch.bfloat16, "cuda", seed=s) for s in (72, 73))
    do = make_tensor((B, H, L, D), torch.bfloat16, "cuda", seed=74)
    (o, dq, dk, dv), lse, _ = _run(rattn, q, k, v, do, cp, 1, True)
    kr, vr = (t.repeat_interleave(H // H_kv, dim=1).contiguous() for t in (k, v))
    qp, pos = rattn.cp_layout_permute(q, cp)
    kp, _ = rattn.cp_layout_permute(kr, cp)
    vp, _ = rattn.cp_layout_permute(vr, cp)
    dop, _ = rattn.cp_layout_permute(do, cp)
    o2, lse2 = rattn.rattn_ring_fwd(qp, kp, vp, pos, cp)
    dq2, dk2, dv2 = rattn.rattn_ring_bwd(qp, kp, vp, o2, dop, lse2, pos, cp)
    torch.cuda.synchronize()
    assert torch.equal(rattn.cp_layout_unpermute(o2, L, cp), o)
    assert torch.equal(lse2, lse)
    # dQ sums per-tile contributions with atomics, in no fixed order
    dq_m = rattn.cp_layout_unpermute(dq2, L, cp).float()
    assert (dq.float() - dq_m).abs().max().item() <= 1e-2 * dq_m.abs().max().item()
    for got, full in ((dk, dk2), (dv, dv2)):
        summed = rattn.cp_layout_unpermute(full, L, cp).float().view(B, H_kv, H // H_kv, L, D).sum(2)
        err = (got.float() - summed).abs().max().item()
        assert err <= 3e-2 * summed.abs().max().item()


def test_ring_gqa_full_size_sampled(rattn):
    """32k tokens / cp=4 with 32 query heads on 8 key/value heads, in the
    launch configuration the bench times: forward on sampled rows of heads
    0, 13 and 31 against the oracle."""
    w = WORKLOADS["bf16_L32000_cp4_gqa8_fwdbwd"]
    q, k, v = make_qkv(w, "cuda", seed=0)
    qp, pos = rattn.cp_layout_permute(q, w.cp, w.layout)
    kp, _ = rattn.cp_layout_permute(k, w.cp, w.layout)
    vp, _ = rattn.cp_layout_permute(v, w.cp, w.layout)
    o, lse = rattn.rattn_ring_fwd_gqa(qp, kp, vp, pos, w.cp, w.layout, True, w.scale, L_valid=w.L)
    torch.cuda.synchronize()
    g = np.random.default_rng(1)
    rows = np.unique(np.concatenate([g.integers(0, w.L, 96), [0, 1, 3999, 4000, 31999]]))
    _, _, pos_ref = oracle.perm_index(w.L, w.cp, w.layout)
    slots = torch.from_numpy(np.argsort(pos_ref)[rows]).cuda()
    group = w.H // w.kv_heads
    for h in (0, 13, 31):
        qh = to64(q[0, h, torch.from_numpy(rows).cuda()])
        kh, vh = to64(k[0, h // group]), to64(v[0, h // group])
        o_ref, l_ref = oracle.attention(qh, kh, vh, w.scale, True, q_pos=rows, kv_pos=np.arange(w.L), row_block=64)
        check_o(o[0, h, slots].float().cpu().numpy(), o_ref, w.torch_dtype)
        check_lse(lse[0, h, slots].cpu().numpy(), l_ref, w.torch_dtype)
