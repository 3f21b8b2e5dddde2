"""GPU parity of the hop-by-hop backward (the calls a ring across processes
makes: rattn_bwd_prep, rattn_partial_bwd, rattn_grad_fold) against the
oracle's share of one key block in the gradient, and of the multi-process
schedules of ``ring_dist`` run on one GPU as a group of one process.

Tolerances are the gradient ones of ``tests/gpu_common.py`` (3e-2 max-abs and
scale-free); Delta is fp32 arithmetic on bf16 inputs (1e-5 relative); the fold
is one fp32 addition per element (bit-exact against torch's)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from context_ring_attention_emulated_b200.workloads import make_tensor
from tests.gpu_common import check_grad, check_lse, check_o, load_rattn, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rattn():
    return load_rattn()


def test_prep_delta_and_accumulator(rattn):
    o = make_tensor((2, 3, 300, 128), torch.bfloat16, "cuda", seed=1)
    do = make_tensor((2, 3, 300, 128), torch.bfloat16, "cuda", seed=2)
    delta, dq = rattn.rattn_bwd_prep(o, do)
    ref = (to64(o) * to64(do)).sum(-1)
    np.testing.assert_allclose(delta.cpu().numpy(), ref, rtol=1e-5, atol=1e-5)
    assert dq.shape == (2, 3, 300, 128) and not dq.any()
    filled = torch.ones(2, 3, 300, 128, device="cuda")
    rattn.rattn_bwd_prep(o, do, dq_acc=filled)
    assert not filled.any()
    d2, none = rattn.rattn_bwd_prep(o, do, dq_acc=None)
    assert none is None and torch.equal(d2, delta)


def _pos(L, cp, layout, r):
    _, _, pos = oracle.perm_index(L, cp, layout)
    n = len(pos) // cp
    return np.asarray(pos[r * n:(r + 1) * n], dtype=np.int32)


# D, H, H_kv, (q positions, kv positions), causal, kv_valid
HT = oracle.HEAD_TAIL
CASES = [
    (128, 2, 2, (_pos(1000, 4, HT, 2), _pos(1000, 4, HT, 1)), True, None),    # s < r: a dense rectangle
    (128, 2, 2, (_pos(1000, 4, HT, 1), _pos(1000, 4, HT, 3)), True, None),    # s > r: tail chunk only
    (128, 2, 2, (_pos(1000, 4, HT, 2), _pos(1000, 4, HT, 2)), True, None),    # the diagonal block
    (64, 4, 2, (np.arange(700, 1000), np.arange(0, 700)), True, None),        # GQA, all visible, Lq != Lk
    (128, 2, 1, (np.arange(129), np.arange(257)), True, None),                 # MQA, ragged tails, causal cut
    (64, 2, 2, (np.arange(200), np.arange(190, 450)), False, 400),             # non-causal, pad keys masked
    (128, 1, 1, (np.arange(0, 100), np.arange(500, 900)), True, None),         # keys all in the future
    (64, 1, 1, (np.arange(0, 140000), np.arange(70000, 70300)), True, None),  # 1094 query tiles: 3-round searches
]


def _inputs(D, H, H_kv, Lq, Lk, seed):
    q = make_tensor((1, H, Lq, D), torch.bfloat16, "cuda", seed=seed)
    do = make_tensor((1, H, Lq, D), torch.bfloat16, "cuda", seed=seed + 1)
    k, v = (make_tensor((1, H_kv, Lk, D), torch.bfloat16, "cuda", seed=seed + s) for s in (2, 3))
    return q, k, v, do


def _row_stats(q, k, v, q_pos, kv_pos, scale, causal, kv_valid, seed):
    """An LSE at or above the block's own (the row's final LSE spans more
    keys) and an arbitrary Delta, both exactly representable in fp32."""
    H = q.shape[1]
    _, lse_blk = oracle.attention(to64(q), oracle.gqa_expand(to64(k), H), oracle.gqa_expand(to64(v), H), scale,
                                  causal, q_pos, kv_pos, kv_valid)
    g = np.random.default_rng(seed)
    lse = np.where(np.isfinite(lse_blk), lse_blk, 0.0) + g.uniform(0.0, 2.0, lse_blk.shape)
    delta = 0.3 * g.standard_normal(lse_blk.shape)
    return np.float32(lse), np.float32(delta)


def _oracle_share(q, k, v, do, lse, delta, q_pos, kv_pos, scale, causal, kv_valid):
    H, H_kv = q.shape[1], k.shape[1]
    dq, dke, dve = oracle.attention_bwd_block(to64(q), oracle.gqa_expand(to64(k), H), oracle.gqa_expand(to64(v), H),
                                              to64(do), lse.astype(np.float64), delta.astype(np.float64), scale,
                                              causal, q_pos, kv_pos, kv_valid)
    return dq, oracle.gqa_reduce(dke, H_kv), oracle.gqa_reduce(dve, H_kv)


@pytest.mark.parametrize("case", range(len(CASES)))
def test_partial_bwd_matches_the_oracle_share(rattn, case):
    D, H, H_kv, (qp, kp), causal, kv_valid = CASES[case]
    Lq, Lk = len(qp), len(kp)
    scale = D ** -0.5
    q, k, v, do = _inputs(D, H, H_kv, Lq, Lk, 10 * case)
    lse, delta = _row_stats(q, k, v, qp, kp, scale, causal, kv_valid, case)
    dq = torch.zeros(1, H, Lq, D, device="cuda")
    q_pos, kv_pos = (torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).cuda() for x in (qp, kp))
    lse_t, delta_t = torch.from_numpy(lse).cuda(), torch.from_numpy(delta).cuda()
    kvv = 2 ** 62 if kv_valid is None else kv_valid
    dk, dv = rattn.rattn_partial_bwd(q, k, v, do, lse_t, delta_t, q_pos, kv_pos, dq, scale, causal, kvv)
    torch.cuda.synchronize()
    assert rattn.rattn_get_device_error()[0] == rattn.OK
    ref = _oracle_share(q, k, v, do, lse, delta, qp, kp, scale, causal, kv_valid)
    for got, want in zip((dq, dk, dv), ref):
        if np.abs(want).max() == 0:
            assert not got.any()
        else:
            check_grad(got.cpu().numpy(), want)
    # accumulate: a second call adds the same shares again
    rattn.rattn_partial_bwd(q, k, v, do, lse_t, delta_t, q_pos, kv_pos, dq, scale, causal, kvv, dk, dv, True)
    for got, want in zip((dq, dk, dv), ref):
        if np.abs(want).max() > 0:
            check_grad(got.cpu().numpy() / 2, want)


def test_partial_bwd_without_query_rows_writes_zero_shares(rattn):
    q = torch.empty(1, 2, 0, 64, dtype=torch.bfloat16, device="cuda")
    k, v = (make_tensor((1, 2, 300, 64), torch.bfloat16, "cuda", seed=s) for s in (5, 6))
    e = torch.empty(1, 2, 0, device="cuda")
    dk = torch.full((1, 2, 300, 64), 7.0, device="cuda")
    dv = torch.full((1, 2, 300, 64), 7.0, device="cuda")
    pos0 = torch.empty(0, dtype=torch.int32, device="cuda")
    kvp = torch.arange(300, dtype=torch.int32, device="cuda")
    rattn.rattn_partial_bwd(q, k, v, q, e, e, pos0, kvp, torch.empty(1, 2, 0, 64, device="cuda"), dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert not dk.any() and not dv.any()


def test_grad_fold_is_one_fp32_addition(rattn):
    a = make_tensor((3, 5, 333, 64), torch.float32, "cuda", seed=7)
    b = make_tensor((3, 5, 333, 64), torch.float32, "cuda", seed=8)
    want = a + b
    rattn.rattn_grad_fold(a, b)
    assert torch.equal(a, want)


def test_four_rank_ring_hop_by_hop_equals_the_gradient(rattn):
    """A cp = 4 head-tail ring, every hop of every rank one rattn_partial_bwd
    call (the shares of each block summed as they would travel), against the
    oracle's gradient of the whole sequence and the emulated ring backward."""
    B, H, L, D, cp = 1, 2, 1000, 128, 4
    scale = D ** -0.5
    q, k, v, do = (make_tensor((B, H, L, D), torch.bfloat16, "cuda", seed=s) for s in (21, 22, 23, 24))
    qp, pos = rattn.cp_layout_permute(q, cp)
    kp, _ = rattn.cp_layout_permute(k, cp)
    vp, _ = rattn.cp_layout_permute(v, cp)
    dop, _ = rattn.cp_layout_permute(do, cp)
    o, lse = rattn.rattn_ring_fwd(qp, kp, vp, pos, cp, L_valid=L)
    n = qp.shape[2] // cp
    sl = lambda x, r: x[:, :, r * n:(r + 1) * n].contiguous()
    dq_all, dk_all, dv_all = [], [None] * cp, [None] * cp
    for r in range(cp):
        delta, dq = rattn.rattn_bwd_prep(sl(o, r), sl(dop, r))
        lse_r = lse[:, :, r * n:(r + 1) * n].contiguous()
        for t in range(cp):
            s = (r - t) % cp
            dk, dv = rattn.rattn_partial_bwd(sl(qp, r), sl(kp, s), sl(vp, s), sl(dop, r), lse_r, delta,
                                             pos[r * n:(r + 1) * n], pos[s * n:(s + 1) * n], dq, scale, True, L)
            if dk_all[s] is None:
                dk_all[s], dv_all[s] = dk, dv
            else:
                rattn.rattn_grad_fold(dk_all[s], dk)
                rattn.rattn_grad_fold(dv_all[s], dv)
        dq_all.append(dq)
    perm = lambda parts: torch.cat(parts, dim=2).contiguous()
    dq_g = rattn.cp_layout_unpermute(perm(dq_all), L, cp)
    dk_g = rattn.cp_layout_unpermute(perm(dk_all), L, cp)
    dv_g = rattn.cp_layout_unpermute(perm(dv_all), L, cp)
    torch.cuda.synchronize()
    assert rattn.rattn_get_device_error()[0] == rattn.OK
    ref = oracle.attention_bwd(to64(q), to64(k), to64(v), to64(do), scale, True)
    for got, want in zip((dq_g, dk_g, dv_g), ref):
        check_grad(got.cpu().numpy(), want)
    # the emulated ring's own backward on the same inputs agrees too
    e_dq, e_dk, e_dv = rattn.rattn_ring_bwd(qp, kp, vp, o, dop, lse, pos, cp, L_valid=L)
    for got, emu in zip((perm(dq_all), perm(dk_all), perm(dv_all)), (e_dq, e_dk, e_dv)):
        check_grad(got.cpu().numpy(), emu.float().cpu().numpy())


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_ring_dist_schedules_on_a_group_of_one(rattn):
    """ring_dist with its default (CUDA kernel) block arithmetic, on a
    one-process group: forward and backward of both exchange options equal
    the oracle's attention of the local rows."""
    from context_ring_attention_emulated_b200 import ring_dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        B, H, L, D = 1, 2, 600, 128
        scale = D ** -0.5
        q, k, v, do = (make_tensor((B, H, L, D), torch.bfloat16, "cuda", seed=s) for s in (31, 32, 33, 34))
        pos = torch.arange(L, dtype=torch.int32, device="cuda")
        o, lse = ring_dist.ring_fwd(q, k, v, pos)
        o2, lse2 = ring_dist.allgather_fwd(q, k, v, pos)
        assert torch.equal(o, o2) and torch.equal(lse, lse2)
        o_ref, lse_ref = oracle.attention(to64(q), to64(k), to64(v), scale, True)
        check_o(o.cpu().numpy(), o_ref, torch.bfloat16)
        check_lse(lse.cpu().numpy(), lse_ref, torch.bfloat16)
        ob = o.to(torch.bfloat16)
        ref = oracle.attention_bwd(to64(q), to64(k), to64(v), to64(do), scale, True)
        for fn in (ring_dist.ring_bwd, ring_dist.allgather_bwd):
            grads = fn(q, k, v, ob, do, lse, pos)
            torch.cuda.synchronize()
            for got, want in zip(grads, ref):
                assert got.dtype == torch.float32
                check_grad(got.cpu().numpy(), want)
    finally:
        dist.destroy_process_group()
