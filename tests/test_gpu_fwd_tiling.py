"""The forms of the bf16 attention forward (one 128-row query tile per CTA;
two sharing each staged K/V tile; a persistent kernel taking one-tile work
items from a per-launch counter; 128 query rows against 256-key tiles) against
each other and the oracle.

The library picks the form by row length and packing; rattn_set_fwd_tiling
forces one. All evaluate every row's online softmax over the same key tiles in
the same order with the same arithmetic, so O and LSE must be bit-identical;
the two-tile results are also checked against the oracle at the bf16
tolerances.
Cases cover odd tile counts (the last pair has no second tile), ragged and
padded lengths, both masks, the striped and contiguous layouts, D = 64,
grouped key/value heads, packed sequences and the partial (one block) call."""
import numpy as np
import pytest
import torch

import oracle
from context_ring_attention_emulated_b200.workloads import make_tensor
from tests.gpu_common import check_lse, check_o, load_rattn, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rattn():
    r = load_rattn()
    yield r
    r.rattn_set_fwd_tiling(0)


def _all_forms(rattn, fn, wide=True):
    """Forms 1-3 bit-identical; form 4 (256-key tiles; D = 128 only) within the
    bf16 tolerances of form 1, since it folds the keys in 256-key steps."""
    outs = []
    for mode in (1, 2, 3):
        rattn.rattn_set_fwd_tiling(mode)
        outs.append([t.clone() for t in fn()])
        torch.cuda.synchronize()
        assert rattn.rattn_get_device_error()[0] == rattn.OK
    if wide:
        rattn.rattn_set_fwd_tiling(4)
        w_o, w_l = (t.clone() for t in fn())
        torch.cuda.synchronize()
        assert rattn.rattn_get_device_error()[0] == rattn.OK
    rattn.rattn_set_fwd_tiling(0)
    for other in outs[1:]:
        for a, b in zip(outs[0], other):
            assert torch.equal(a, b), "the tilings differ"
    if wide:
        ref_o, ref_l = (t.float() for t in outs[0])
        assert ((w_o.float() - ref_o).abs() <= 2e-2 + 1e-2 * ref_o.abs()).all()
        fin = torch.isfinite(ref_l)
        assert torch.equal(fin, torch.isfinite(w_l))
        assert (w_l[fin] - ref_l[fin]).abs().max().item() <= 1e-3 if fin.any() else True
    return outs[1]


RING = [
    # B, H, H_kv, L, D, cp, layout, causal
    (1, 2, 2, 1000, 128, 2, 1, True),     # 500-row slices: 4 tiles, a ragged last one
    (1, 4, 2, 2000, 128, 4, 1, True),     # GQA
    (2, 2, 2, 777, 64, 3, 1, True),       # padded to 780, 3 tiles a slice, D = 64
    (1, 2, 1, 1500, 128, 4, 2, True),     # striped, MQA, 3 tiles a slice
    (1, 2, 2, 1300, 128, 2, 0, False),    # contiguous, non-causal
    (1, 1, 1, 8192, 128, 2, 1, True),     # 32 tiles per slice
    (1, 2, 2, 1664, 128, 2, 1, True),     # 832-row slices: 7 tiles, an odd count
    (1, 2, 2, 640, 64, 1, 0, True),       # one rank: 5 tiles, D = 64
    (1, 2, 2, 3000, 128, 64, 1, True),    # 64 ranks (the most a call takes): 64 hops per tile
]


@pytest.mark.parametrize("case", RING)
def test_ring_fwd_tilings_agree_and_match_oracle(rattn, case):
    B, H, H_kv, L, D, cp, layout, causal = case
    scale = D ** -0.5
    q = make_tensor((B, H, L, D), torch.bfloat16, "cuda", seed=61)
    k, v = (make_tensor((B, H_kv, L, D), torch.bfloat16, "cuda", seed=s) for s in (62, 63))
    qp, pos = rattn.cp_layout_permute(q, cp, layout)
    kp, _ = rattn.cp_layout_permute(k, cp, layout)
    vp, _ = rattn.cp_layout_permute(v, cp, layout)
    fwd = rattn.rattn_ring_fwd_gqa if H_kv != H else rattn.rattn_ring_fwd
    o, lse = _all_forms(rattn, lambda: fwd(qp, kp, vp, pos, cp, layout, causal, scale, L_valid=L),
                        wide=D == 128 and cp <= 32)
    out = rattn.cp_layout_unpermute(o, L, cp, layout)
    ke, ve = oracle.gqa_expand(to64(k), H), oracle.gqa_expand(to64(v), H)
    o_ref, l_ref = oracle.attention(to64(q), ke, ve, scale, causal)
    check_o(out.float().cpu().numpy(), o_ref, torch.bfloat16)
    real = pos.cpu().numpy() < L
    l_ref_p, _ = oracle.permute(l_ref[..., None], cp, layout)
    check_lse(lse.cpu().numpy()[..., real], l_ref_p[..., 0][..., real], torch.bfloat16)


GROWING = [
    # L, cp, layout, causal, drift of the scores along the keys (natural-log units)
    (4096, 2, 1, True, 60.0),
    (4096, 4, 0, False, 60.0),
    (4096, 2, 1, True, -60.0),
    (3000, 3, 2, True, 90.0),
]


@pytest.mark.parametrize("case", GROWING)
def test_ring_fwd_scores_that_drift(rattn, case):
    """Scores rising (or falling) by tens of natural-log units along the keys
    (q ~ 1, k_j ~ t_j / sqrt(D), so q.k_j scale ~ t_j): a row's running max
    moves many times across its tiles, which exercises every form's lazy
    rescale and the 256-key form's short path handing over to its full path.
    All forms against the oracle, the 256-key one (the default) included."""
    L, cp, layout, causal, drift = case
    B, H, D = 1, 2, 128
    scale = D ** -0.5
    t = drift * torch.arange(L, dtype=torch.float32, device="cuda") / L
    q = (1.0 + 0.05 * make_tensor((B, H, L, D), torch.float32, "cuda", seed=101)).to(torch.bfloat16)
    k = (t[None, None, :, None] * scale + 0.05 * make_tensor((B, H, L, D), torch.float32, "cuda", seed=102))
    k = k.to(torch.bfloat16)
    v = make_tensor((B, H, L, D), torch.bfloat16, "cuda", seed=103)
    qp, pos = rattn.cp_layout_permute(q, cp, layout)
    kp, _ = rattn.cp_layout_permute(k, cp, layout)
    vp, _ = rattn.cp_layout_permute(v, cp, layout)
    run = lambda: rattn.rattn_ring_fwd(qp, kp, vp, pos, cp, layout, causal, scale, L_valid=L)
    _all_forms(rattn, run)
    o_ref, l_ref = oracle.attention(to64(q), to64(k), to64(v), scale, causal)
    l_ref_p, _ = oracle.permute(l_ref[..., None], cp, layout)
    real = pos.cpu().numpy() < L
    for mode in (1, 4):
        rattn.rattn_set_fwd_tiling(mode)
        o, lse = run()
        torch.cuda.synchronize()
        rattn.rattn_set_fwd_tiling(0)
        assert rattn.rattn_get_device_error()[0] == rattn.OK
        out = rattn.cp_layout_unpermute(o, L, cp, layout)
        check_o(out.float().cpu().numpy(), o_ref, torch.bfloat16)
        check_lse(lse.cpu().numpy()[..., real], l_ref_p[..., 0][..., real], torch.bfloat16)


def test_partial_fwd_tilings_agree(rattn):
    """One block with separate query and key positions, masked pad keys, and
    an empty key block."""
    q = make_tensor((1, 2, 700, 128), torch.bfloat16, "cuda", seed=71)
    k, v = (make_tensor((1, 2, 900, 128), torch.bfloat16, "cuda", seed=s) for s in (72, 73))
    qpos = np.arange(200, 900, dtype=np.int32)
    kpos = np.arange(0, 900, dtype=np.int32)
    qd, kd = torch.from_numpy(qpos).cuda(), torch.from_numpy(kpos).cuda()
    o, lse = _all_forms(rattn, lambda: rattn.rattn_partial_fwd(q, k, v, qd, kd, causal=True, kv_valid=850))
    o_ref, l_ref = oracle.attention(to64(q), to64(k), to64(v), 128 ** -0.5, True, qpos, kpos, 850)
    check_lse(lse.cpu().numpy(), l_ref, torch.bfloat16)
    check_o(o.cpu().numpy(), o_ref, torch.bfloat16)
    e_k = torch.empty(1, 2, 0, 128, dtype=torch.bfloat16, device="cuda")
    o0, l0 = _all_forms(rattn, lambda: rattn.rattn_partial_fwd(q, e_k, e_k, causal=True))
    assert torch.all(o0 == 0) and torch.all(torch.isneginf(l0))


def test_partial_fwd_tilings_agree_on_long_key_blocks(rattn):
    """More than 1024 key tiles per block (three rounds of the tile-range
    searches), causal with the query rows in the middle of the keys."""
    q = make_tensor((1, 1, 300, 64), torch.bfloat16, "cuda", seed=74)
    k, v = (make_tensor((1, 1, 140000, 64), torch.bfloat16, "cuda", seed=s) for s in (75, 76))
    qpos = np.arange(70000, 70300, dtype=np.int32)
    kpos = np.arange(0, 140000, dtype=np.int32)
    qd, kd = torch.from_numpy(qpos).cuda(), torch.from_numpy(kpos).cuda()
    o, lse = _all_forms(rattn, lambda: rattn.rattn_partial_fwd(q, k, v, qd, kd, causal=True), wide=False)
    o_ref, l_ref = oracle.attention(to64(q), to64(k), to64(v), 64 ** -0.5, True, qpos, kpos)
    check_lse(lse.cpu().numpy(), l_ref, torch.bfloat16)
    check_o(o.cpu().numpy(), o_ref, torch.bfloat16)


def test_packed_fwd_tilings_agree(rattn):
    cu = [0, 5, 300, 301, 1000, 1900]
    cp = 2
    plan = rattn.cp_layout_varlen_plan(cu, cp, 1, 128)
    src, gkey, segid = (plan[n].cuda() for n in ("src", "gkey", "segid"))
    q, k, v = (make_tensor((1, 2, cu[-1], 128), torch.bfloat16, "cuda", seed=s) for s in (81, 82, 83))
    qp, kp, vp = (rattn.cp_layout_gather(t, src) for t in (q, k, v))
    o, lse = _all_forms(rattn, lambda: rattn.rattn_ring_fwd_varlen(qp, kp, vp, gkey, segid, cp, True))
    out = rattn.cp_layout_scatter(o, src, cu[-1])
    for a, b in zip(cu, cu[1:]):
        if a == b:
            continue
        o_ref, _ = oracle.attention(to64(q[..., a:b, :]), to64(k[..., a:b, :]), to64(v[..., a:b, :]),
                                    128 ** -0.5, True)
        check_o(out[..., a:b, :].float().cpu().numpy(), o_ref, torch.bfloat16)


def test_persistent_work_counters_reset_between_launches(rattn):
    """Persistent launches back to back on one stream (sizes from one work
    item per CTA to many, and one with no visible key at all), then two at
    once on two streams: every launch must take each of its work items
    exactly once, or its rows would be missing or stale."""
    shapes = [(1, 1, 300, 300), (2, 4, 3000, 3000), (1, 2, 700, 0), (1, 8, 5000, 5000), (1, 1, 130, 130)]
    inputs, refs = [], []
    rattn.rattn_set_fwd_tiling(1)
    try:
        for i, (B, H, Lq, Lk) in enumerate(shapes):
            q = make_tensor((B, H, Lq, 128), torch.bfloat16, "cuda", seed=90 + i)
            k, v = (make_tensor((B, H, Lk, 128), torch.bfloat16, "cuda", seed=95 + i + j) for j in (0, 7))
            inputs.append((q, k, v))
            refs.append([t.clone() for t in rattn.rattn_partial_fwd(q, k, v, causal=True)])
        rattn.rattn_set_fwd_tiling(3)
        for rep in range(2):
            outs = [rattn.rattn_partial_fwd(q, k, v, causal=True) for q, k, v in inputs]
            torch.cuda.synchronize()
            for got, want in zip(outs, refs):
                assert torch.equal(got[0], want[0]) and torch.equal(got[1], want[1])
        s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
        torch.cuda.synchronize()
        with torch.cuda.stream(s1):
            a = rattn.rattn_partial_fwd(*inputs[1], causal=True)
        with torch.cuda.stream(s2):
            b = rattn.rattn_partial_fwd(*inputs[3], causal=True)
        torch.cuda.synchronize()
        assert torch.equal(a[0], refs[1][0]) and torch.equal(b[0], refs[3][0])
        assert rattn.rattn_get_device_error()[0] == rattn.OK
    finally:
        rattn.rattn_set_fwd_tiling(0)
