"""The deterministic mode of the ring backward (rattn_set_bwd_deterministic):
dQ from the query-stationary pass. Checked against the oracle's textbook
softmax-attention gradient at the gradient tolerances, against the default
mode's dQ (the same gradient up to accumulation order), and for bit-identical
dQ, dK, dV across repeated runs, including a full-size 32k / cp=4 run where
the default mode's fp32 reduce-adds land in a different order every time."""
import pytest
import torch

import oracle
from context_ring_attention_emulated_b200.workloads import WORKLOADS, make_qkv, make_tensor
from tests.gpu_common import check_grad, load_rattn, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rattn():
    r = load_rattn()
    yield r
    r.rattn_set_bwd_deterministic(False)


def _grads(rattn, q, k, v, do, cp, layout, causal, deterministic, fwd=None):
    L, D = q.shape[2], q.shape[3]
    H, H_kv = q.shape[1], k.shape[1]
    qp, pos = rattn.cp_layout_permute(q, cp, layout)
    kp, _ = rattn.cp_layout_permute(k, cp, layout)
    vp, _ = rattn.cp_layout_permute(v, cp, layout)
    dop, _ = rattn.cp_layout_permute(do, cp, layout)
    gqa = H_kv != H
    ring_fwd = rattn.rattn_ring_fwd_gqa if gqa else rattn.rattn_ring_fwd
    ring_bwd = rattn.rattn_ring_bwd_gqa if gqa else rattn.rattn_ring_bwd
    o, lse = ring_fwd(qp, kp, vp, pos, cp, layout, causal, D ** -0.5, L_valid=L)
    rattn.rattn_set_bwd_deterministic(deterministic)
    try:
        dq, dk, dv = ring_bwd(qp, kp, vp, o, dop, lse, pos, cp, layout, causal, D ** -0.5, L_valid=L)
        torch.cuda.synchronize()
    finally:
        rattn.rattn_set_bwd_deterministic(False)
    assert rattn.rattn_get_device_error()[0] == rattn.OK
    return [rattn.cp_layout_unpermute(g, L, cp, layout) for g in (dq, dk, dv)]


CASES = [
    # D, L, cp, layout, causal, H, H_kv
    (128, 1000, 4, 1, True, 2, 2),     # head-tail, ragged last tile
    (64, 777, 3, 1, True, 2, 2),       # padded, D = 64
    (128, 1300, 2, 0, False, 2, 2),    # contiguous, non-causal, pad keys masked
    (128, 1500, 4, 2, True, 2, 2),     # striped
    (128, 2000, 4, 1, True, 4, 2),     # GQA
    (64, 3000, 64, 1, True, 1, 1),     # 64 ranks
]


@pytest.mark.parametrize("case", CASES)
def test_deterministic_bwd_matches_oracle_and_repeats(rattn, case):
    D, L, cp, layout, causal, H, H_kv = case
    q = make_tensor((1, H, L, D), torch.bfloat16, "cuda", seed=41)
    k, v = (make_tensor((1, H_kv, L, D), torch.bfloat16, "cuda", seed=s) for s in (42, 43))
    do = make_tensor((1, H, L, D), torch.bfloat16, "cuda", seed=44)
    det = _grads(rattn, q, k, v, do, cp, layout, causal, True)
    again = _grads(rattn, q, k, v, do, cp, layout, causal, True)
    for a, b in zip(det, again):
        assert torch.equal(a, b), "deterministic mode gave different bits"
    dflt = _grads(rattn, q, k, v, do, cp, layout, causal, False)
    assert torch.equal(det[1], dflt[1]) and torch.equal(det[2], dflt[2])  # dK, dV: the same kernel
    ke, ve = oracle.gqa_expand(to64(k), H), oracle.gqa_expand(to64(v), H)
    dq_ref, dk_ref, dv_ref = oracle.attention_bwd(to64(q), ke, ve, to64(do), D ** -0.5, causal)
    check_grad(det[0].float().cpu().numpy(), dq_ref)
    check_grad(det[1].float().cpu().numpy(), oracle.gqa_reduce(dk_ref, H_kv))
    check_grad(det[2].float().cpu().numpy(), oracle.gqa_reduce(dv_ref, H_kv))
    # the two modes' dQ: one gradient, summed in two orders
    diff = (det[0].float() - dflt[0].float()).abs().max().item()
    assert diff <= 3e-2 * max(dq_ref.__abs__().max(), 1e-30)


def test_deterministic_packed_bwd(rattn):
    cu = [0, 5, 300, 301, 1000, 1900]
    cp, T = 2, 1900
    plan = rattn.cp_layout_varlen_plan(cu, cp, 1, 128)
    src, gkey, segid = (plan[n].cuda() for n in ("src", "gkey", "segid"))
    q, k, v, do = (make_tensor((1, 2, T, 128), torch.bfloat16, "cuda", seed=s) for s in (51, 52, 53, 54))
    qp, kp, vp, dop = (rattn.cp_layout_gather(t, src) for t in (q, k, v, do))
    o, lse = rattn.rattn_ring_fwd_varlen(qp, kp, vp, gkey, segid, cp, True)
    outs = []
    for _ in range(2):
        rattn.rattn_set_bwd_deterministic(True)
        try:
            g = rattn.rattn_ring_bwd_varlen(qp, kp, vp, o, dop, lse, gkey, segid, cp, True)
            torch.cuda.synchronize()
        finally:
            rattn.rattn_set_bwd_deterministic(False)
        outs.append([t.clone() for t in g])
    for a, b in zip(*outs):
        assert torch.equal(a, b)
    dq = rattn.cp_layout_scatter(outs[0][0], src, T)
    for a, b in zip(cu, cu[1:]):
        if a == b:
            continue
        ref, _, _ = oracle.attention_bwd(to64(q[..., a:b, :]), to64(k[..., a:b, :]), to64(v[..., a:b, :]),
                                         to64(do[..., a:b, :]), 128 ** -0.5, True)
        check_grad(dq[..., a:b, :].float().cpu().numpy(), ref)


def test_deterministic_bwd_full_size_repeats_bit_for_bit(rattn):
    """32k tokens / cp=4, 8 heads: three deterministic runs give the same
    bits; dQ agrees with the default mode's to the gradient tolerance."""
    w = WORKLOADS["bf16_L32000_cp4_fwdbwd"]
    q, k, v = (t[:, :8].contiguous() for t in make_qkv(w, "cuda", seed=0))
    do = make_tensor(q.shape, q.dtype, "cuda", seed=1)
    runs = [_grads(rattn, q, k, v, do, w.cp, w.layout, True, True) for _ in range(3)]
    for other in runs[1:]:
        for a, b in zip(runs[0], other):
            assert torch.equal(a, b)
    dflt = _grads(rattn, q, k, v, do, w.cp, w.layout, True, False)
    ref_max = dflt[0].float().abs().max().item()
    assert (runs[0][0].float() - dflt[0].float()).abs().max().item() <= 3e-2 * ref_max
