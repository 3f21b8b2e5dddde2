"""Pins for the oracle's attention, merge, ring and gradient (CPU only).

Each pin fixes the oracle to something other than itself: brute force with
Python loops and math.exp, closed forms, a library special case (torch's fp64
CPU scaled_dot_product_attention and autograd), central finite differences,
and the ring invariant the pages state (blockwise online softmax over any
chunking equals full attention). A last test plants plausible mistakes in a
copy of the oracle and checks that these pins reject every one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import attn as oatt

RNG = np.random.default_rng(12345)


def brute_attention(q, k, v, scale, causal, q_pos, kv_pos, kv_valid=None):
    """Python loops over rows and keys, math.exp, no numpy arithmetic."""
    Lq, D = q.shape
    Lk = k.shape[0]
    O = [[0.0] * v.shape[1] for _ in range(Lq)]
    lse = [0.0] * Lq
    for i in range(Lq):
        vis = [j for j in range(Lk)
               if (not causal or kv_pos[j] <= q_pos[i]) and (kv_valid is None or kv_pos[j] < kv_valid)]
        if not vis:
            lse[i] = -math.inf
            continue
        s = {j: scale * sum(float(q[i, d]) * float(k[j, d]) for d in range(D)) for j in vis}
        mx = max(s.values())
        w = {j: math.exp(s[j] - mx) for j in vis}
        tot = sum(w.values())
        lse[i] = mx + math.log(tot)
        for e in range(v.shape[1]):
            O[i][e] = sum(w[j] * float(v[j, e]) for j in vis) / tot
    return np.array(O), np.array(lse)


def _case(Lq, Lk, D, seed):
    r = np.random.default_rng(seed)
    return r.standard_normal((Lq, D)), r.standard_normal((Lk, D)), r.standard_normal((Lk, D))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Lq,Lk,D", [(1, 1, 1), (3, 5, 2), (8, 8, 4), (6, 7, 3)])
def test_matches_brute_force(causal, Lq, Lk, D):
    q, k, v = _case(Lq, Lk, D, Lq * 100 + Lk * 10 + D)
    r = np.random.default_rng(7)
    q_pos = np.sort(r.integers(0, 10, Lq))
    kv_pos = np.sort(r.integers(0, 10, Lk))
    for kv_valid in (None, 6):
        o, lse = oracle.attention(q, k, v, 0.7, causal, q_pos, kv_pos, kv_valid, row_block=2)
        ob, lb = brute_attention(q, k, v, 0.7, causal, q_pos, kv_pos, kv_valid)
        assert np.array_equal(np.isinf(lse), np.isinf(lb))
        fin = np.isfinite(lb)
        np.testing.assert_allclose(lse[fin], lb[fin], rtol=0, atol=1e-12)
        np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_sdpa_fp64(causal):
    B, H, L, D = 2, 3, 37, 16
    q, k, v = (RNG.standard_normal((B, H, L, D)) for _ in range(3))
    scale = 1.0 / math.sqrt(D)
    o, lse = oracle.attention(q, k, v, scale, causal, row_block=8)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
        ot = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
    s = scale * tq @ tk.transpose(-1, -2)
    if causal:
        s = s.masked_fill(torch.ones(L, L, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(o, ot.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), rtol=0, atol=1e-12)


def test_closed_forms():
    L, D = 9, 5
    _, k, v = _case(L, L, D, 3)
    q0 = np.zeros((L, D))
    o, lse = oracle.attention(q0, k, v, 0.3, True)
    for i in range(L):                           # Q = 0: uniform over visible keys
        np.testing.assert_allclose(o[i], v[:i + 1].mean(axis=0), atol=1e-13)
        assert abs(lse[i] - math.log(i + 1)) < 1e-13
    q, k, _ = _case(L, L, D, 4)
    const = np.tile(np.array([1.5, -2.0, 0.25, 3.0, -0.5]), (L, 1))
    o, _ = oracle.attention(q, k, const, 0.3, False)
    np.testing.assert_allclose(o, const, atol=1e-13)          # constant V
    o, lse = oracle.attention(q[:1], k[:1], v[:1], 0.3, False)
    np.testing.assert_allclose(o[0], v[0], atol=1e-15)       # L = 1
    assert abs(lse[0] - 0.3 * float(q[0] @ k[0])) < 1e-13
    o, lse = oracle.attention(q, k, v, 0.3, True)
    np.testing.assert_allclose(o[0], v[0], atol=1e-15)       # causal row 0 sees only key 0
    assert abs(lse[0] - 0.3 * float(q[0] @ k[0])) < 1e-13


def test_lse_bounds_and_fully_masked_rows():
    q, k, v = _case(12, 12, 4, 9)
    q_pos = np.arange(12)
    kv_pos = np.arange(12) + 3          # rows 0..2 see nothing under causal
    o, lse = oracle.attention(q, k, v, 0.5, True, q_pos, kv_pos)
    assert np.all(np.isneginf(lse[:3])) and np.all(o[:3] == 0.0)
    s = 0.5 * q @ k.T
    for i in range(3, 12):
        vis = kv_pos <= q_pos[i]
        mx = s[i, vis].max()
        assert mx - 1e-12 <= lse[i] <= mx + math.log(vis.sum()) + 1e-12


def test_merge_properties():
    shape = (3, 4)
    oa, ob, oc = (RNG.standard_normal(shape + (5,)) for _ in range(3))
    la, lb, lc = (RNG.standard_normal(shape) * 3 for _ in range(3))
    ninf = np.full(shape, -np.inf)
    o, l = oracle.merge(oa, la, np.zeros_like(oa), ninf)
    np.testing.assert_allclose(o, oa, atol=1e-15)
    np.testing.assert_allclose(l, la, atol=1e-15)
    o, l = oracle.merge(np.zeros_like(oa), ninf, np.zeros_like(oa), ninf)
    assert np.all(np.isneginf(l)) and np.all(o == 0.0) and not np.isnan(o).any()
    o1, l1 = oracle.merge(oa, la, ob, lb)
    o2, l2 = oracle.merge(ob, lb, oa, la)
    np.testing.assert_allclose(o1, o2, atol=1e-14)
    np.testing.assert_allclose(l1, l2, atol=1e-14)
    o3, l3 = oracle.merge(*oracle.merge(oa, la, ob, lb), oc, lc)
    o4, l4 = oracle.merge(oa, la, *oracle.merge(ob, lb, oc, lc))
    np.testing.assert_allclose(o3, o4, atol=1e-13)
    np.testing.assert_allclose(l3, l4, atol=1e-13)
    # two halves of a key set merge to the whole
    q, k, v = _case(6, 10, 3, 21)
    oh1, lh1 = oracle.attention(q, k[:4], v[:4], 0.8, False)
    oh2, lh2 = oracle.attention(q, k[4:], v[4:], 0.8, False)
    of, lf = oracle.attention(q, k, v, 0.8, False)
    om, lm = oracle.merge(oh1, lh1, oh2, lh2)
    np.testing.assert_allclose(om, of, atol=1e-13)
    np.testing.assert_allclose(lm, lf, atol=1e-13)


@pytest.mark.parametrize("trial", range(6))
def test_blockwise_any_chunking_equals_full(trial):
    r = np.random.default_rng(100 + trial)
    L, D = int(r.integers(5, 40)), int(r.integers(1, 6))
    q, k, v = (r.standard_normal((2, L, D)) for _ in range(3))
    causal = bool(trial % 2)
    cuts = np.sort(r.choice(np.arange(1, L), size=min(L - 1, int(r.integers(1, 6))), replace=False))
    blocks = np.split(np.arange(L), cuts)
    order = r.permutation(len(blocks))
    o, lse = oracle.blockwise_attention(q, k, v, 0.4, causal, [blocks[i] for i in order])
    of, lf = oracle.attention(q, k, v, 0.4, causal)
    np.testing.assert_allclose(o, of, atol=1e-12)
    np.testing.assert_allclose(lse, lf, atol=1e-12)


@pytest.mark.parametrize("cp", [1, 2, 3, 4])
@pytest.mark.parametrize("layout", [oracle.HEAD_TAIL, oracle.CONTIGUOUS, oracle.STRIPED])
@pytest.mark.parametrize("causal", [True, False])
def test_ring_equals_full_and_is_layout_invariant(cp, layout, causal):
    L, D = 29, 4
    r = np.random.default_rng(cp * 10 + layout)
    q, k, v = (r.standard_normal((1, 2, L, D)) for _ in range(3))
    (qp, pos), (kp, _), (vp, _) = (oracle.permute(x, cp, layout) for x in (q, k, v))
    o, lse = oracle.ring_emulate(qp, kp, vp, pos, cp, 0.5, causal, kv_valid=L)
    of, lf = oracle.attention(q, k, v, 0.5, causal)
    np.testing.assert_allclose(oracle.unpermute(o, L, cp, layout), of, atol=1e-12)
    lse_u = oracle.unpermute(lse[..., None], L, cp, layout)[..., 0]
    np.testing.assert_allclose(lse_u, lf, atol=1e-12)
    # direct attention on the permuted arrays with carried positions agrees too
    od, ld = oracle.attention(qp, kp, vp, 0.5, causal, pos, pos, kv_valid=L)
    real = pos < L
    np.testing.assert_allclose(o[..., real, :], od[..., real, :], atol=1e-12)
    np.testing.assert_allclose(lse[..., real], ld[..., real], atol=1e-12)


def _fd_grads(q, k, v, do, scale, causal, q_pos, kv_pos, h=1e-6):
    def loss(qq, kk, vv):
        o, _ = oracle.attention(qq, kk, vv, scale, causal, q_pos, kv_pos)
        return float((o * do).sum())
    grads = []
    for which in range(3):
        base = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(base[which])
        for idx in np.ndindex(g.shape):
            plus = [x.copy() for x in base]
            minus = [x.copy() for x in base]
            plus[which][idx] += h
            minus[which][idx] -= h
            g[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        grads.append(g)
    return grads


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("Lq,Lk,D", [(5, 5, 2), (7, 9, 3), (16, 16, 4)])
def test_bwd_matches_finite_differences(causal, Lq, Lk, D):
    r = np.random.default_rng(Lq + Lk + D)
    q, k, v, do = r.standard_normal((Lq, D)), r.standard_normal((Lk, D)), r.standard_normal((Lk, D)), r.standard_normal((Lq, D))
    q_pos = np.arange(Lq) + (Lk - Lq)
    kv_pos = np.arange(Lk)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, 0.6, causal, q_pos, kv_pos, row_block=3)
    for got, ref in zip((dq, dk, dv), _fd_grads(q, k, v, do, 0.6, causal, q_pos, kv_pos)):
        np.testing.assert_allclose(got, ref, rtol=1e-7, atol=1e-8)


@pytest.mark.parametrize("causal", [True, False])
def test_bwd_matches_torch_autograd_fp64(causal):
    B, H, L, D = 1, 2, 33, 8
    q, k, v, do = (RNG.standard_normal((B, H, L, D)) for _ in range(4))
    scale = 1 / math.sqrt(D)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, scale, causal, row_block=10)
    tq, tk, tv = (torch.from_numpy(x).requires_grad_(True) for x in (q, k, v))
    with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
        o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
    o.backward(torch.from_numpy(do))
    for got, ref in zip((dq, dk, dv), (tq.grad, tk.grad, tv.grad)):
        np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-12)


# ---- grouped key/value heads (GQA) ------------------------------------------

@pytest.mark.parametrize("H,H_kv", [(4, 2), (6, 3), (4, 1), (3, 3)])
@pytest.mark.parametrize("causal", [True, False])
def test_gqa_matches_torch_sdpa_enable_gqa(H, H_kv, causal):
    """torch's SDPA with enable_gqa=True (fp64, math backend) and its autograd
    against the oracle's attention on expanded K/V heads and the gradient
    reduced over each group."""
    B, L, D = 2, 21, 8
    q, do = (RNG.standard_normal((B, H, L, D)) for _ in range(2))
    k, v = (RNG.standard_normal((B, H_kv, L, D)) for _ in range(2))
    scale = 0.4
    ke, ve = oracle.gqa_expand(k, H), oracle.gqa_expand(v, H)
    o, lse = oracle.attention(q, ke, ve, scale, causal, row_block=5)
    dq, dke, dve = oracle.attention_bwd(q, ke, ve, do, scale, causal, row_block=5)
    dk, dv = oracle.gqa_reduce(dke, H_kv), oracle.gqa_reduce(dve, H_kv)
    tq, tk, tv = (torch.from_numpy(x).requires_grad_(True) for x in (q, k, v))
    with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
        ot = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale,
                                                              enable_gqa=True)
    ot.backward(torch.from_numpy(do))
    np.testing.assert_allclose(o, ot.detach().numpy(), rtol=0, atol=1e-12)
    for got, ref in zip((dq, dk, dv), (tq.grad, tk.grad, tv.grad)):
        assert got.shape == ref.shape
        np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-12)


def test_gqa_group_membership_and_identity():
    k = RNG.standard_normal((1, 3, 4, 2))
    e = oracle.gqa_expand(k, 6)
    for h in range(6):
        assert np.array_equal(e[0, h], k[0, h // 2])      # contiguous groups of 2
    assert np.array_equal(oracle.gqa_expand(k, 3), k)
    assert np.array_equal(oracle.gqa_reduce(e, 3), 2 * k)  # each head counted once per group member
    with pytest.raises(ValueError):
        oracle.gqa_expand(k, 4)


# ---- the pins catch planted mistakes ---------------------------------------

_ORIG_2D = oatt._attention_2d


def _drop_scale(q, k, v, scale, mask):
    return _ORIG_2D(q, k, v, 1.0, mask)


def _strict_causal(q, k, v, scale, mask):
    m2 = mask.copy()
    for i in range(min(m2.shape)):
        m2[i, i] = False
    return _ORIG_2D(q, k, v, scale, m2)


def _rows_swapped(q, k, v, scale, mask):
    o, lse = _ORIG_2D(q, k, v, scale, mask)
    return o[::-1].copy(), lse


def _log2_normaliser(q, k, v, scale, mask):
    o, lse = _ORIG_2D(q, k, v, scale, mask)
    return o, lse / math.log(2.0)


def _k_for_v(q, k, v, scale, mask):
    return _ORIG_2D(q, k, k, scale, mask)


@pytest.mark.parametrize("mutant", [_drop_scale, _strict_causal, _rows_swapped, _log2_normaliser, _k_for_v])
def test_pins_reject_planted_mistakes(mutant, monkeypatch):
    monkeypatch.setattr(oatt, "_attention_2d", mutant)
    q, k, v = _case(6, 6, 3, 77)
    pos = np.arange(6)
    o, lse = oracle.attention(q, k, v, 0.7, True, pos, pos)
    ob, lb = brute_attention(q, k, v, 0.7, True, pos, pos)
    ok = np.allclose(o, ob, atol=1e-12) and np.allclose(lse, lb, atol=1e-12)
    assert not ok, "a planted mistake passed the brute-force pin"


def test_empty_key_block_sees_nothing():
    q = np.ones((2, 3, 4, 5))
    k = np.zeros((2, 3, 0, 5))
    o, lse = oracle.attention(q, k, k, 0.5, False)
    assert o.shape == (2, 3, 4, 5) and np.all(o == 0.0) and np.all(np.isneginf(lse))
    dq, dk, dv = oracle.attention_bwd(q, k, k, q, 0.5, True)
    assert np.all(dq == 0.0) and dk.shape == k.shape and dv.shape == k.shape


# ---- one hop of the ring backward -------------------------------------------

def _block_bwd_case(seed, causal, kv_valid):
    """Random rows with shuffled (not monotone) positions, the final O / LSE of
    the whole key set, and a random split of the keys into blocks."""
    r = np.random.default_rng(seed)
    B, H, Lq, Lk, D = 2, 2, 11, 13, 4
    q, do = r.standard_normal((B, H, Lq, D)), r.standard_normal((B, H, Lq, D))
    k, v = r.standard_normal((B, H, Lk, D)), r.standard_normal((B, H, Lk, D))
    q_pos = r.permutation(Lq) + 3
    kv_pos = r.permutation(Lk)
    cuts = np.sort(r.choice(np.arange(1, Lk), size=3, replace=False))
    perm = r.permutation(Lk)
    blocks = [np.sort(b) for b in np.split(perm, cuts)]
    o, lse = oracle.attention(q, k, v, 0.45, causal, q_pos, kv_pos, kv_valid, row_block=4)
    delta = (do * o).sum(-1)
    return q, k, v, do, lse, delta, q_pos, kv_pos, blocks


def _sum_of_block_shares(case, causal, kv_valid, block_fn=None):
    q, k, v, do, lse, delta, q_pos, kv_pos, blocks = case
    fn = block_fn or oracle.attention_bwd_block
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for idx in blocks:
        gq, gk, gv = fn(q, k[..., idx, :], v[..., idx, :], do, lse, delta, 0.45, causal, q_pos, kv_pos[idx],
                        kv_valid)
        dq += gq
        dk[..., idx, :] = gk
        dv[..., idx, :] = gv
    return dq, dk, dv


@pytest.mark.parametrize("causal,kv_valid", [(True, None), (False, None), (True, 9), (False, 7)])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_block_bwd_shares_sum_to_the_gradient(causal, kv_valid, seed):
    """Summed over any split of the keys (and keys of each block written back
    in place), the per-block shares are the full gradient (pinned above by
    finite differences and torch autograd): sum_j P_ij dP_ij = delta_i."""
    case = _block_bwd_case(seed, causal, kv_valid)
    q, k, v, do, lse, delta, q_pos, kv_pos, _ = case
    ref = oracle.attention_bwd(q, k, v, do, 0.45, causal, q_pos, kv_pos, kv_valid, row_block=4)
    for got, want in zip(_sum_of_block_shares(case, causal, kv_valid), ref):
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_block_bwd_single_block_matches_finite_differences():
    r = np.random.default_rng(5)
    q, k, v, do = (r.standard_normal((6, 3)) for _ in range(4))
    pos = np.arange(6)
    o, lse = oracle.attention(q, k, v, 0.6, True, pos, pos)
    got = oracle.attention_bwd_block(q, k, v, do, lse, (do * o).sum(-1), 0.6, True, pos, pos)
    for g, ref in zip(got, _fd_grads(q, k, v, do, 0.6, True, pos, pos)):
        np.testing.assert_allclose(g, ref, rtol=1e-7, atol=1e-8)


def test_block_bwd_block_without_visible_keys_is_zero():
    """A block that lies wholly in the future of every query adds nothing."""
    r = np.random.default_rng(6)
    q, do = r.standard_normal((1, 4, 2)), r.standard_normal((1, 4, 2))
    k, v = r.standard_normal((1, 3, 2)), r.standard_normal((1, 3, 2))
    lse = r.standard_normal((1, 4))
    dq, dk, dv = oracle.attention_bwd_block(q, k, v, do, lse, r.standard_normal((1, 4)), 0.5, True,
                                            np.arange(4), np.arange(10, 13))
    assert not dq.any() and not dk.any() and not dv.any()


def _delta_dropped(q, k, v, do, lse, delta, *a):
    return oracle.attention_bwd_block(q, k, v, do, lse, np.zeros_like(delta), *a)


def _lse_base2(q, k, v, do, lse, delta, *a):
    return oracle.attention_bwd_block(q, k, v, do, lse / math.log(2.0), delta, *a)


def _v_for_k(q, k, v, do, lse, delta, *a):
    return oracle.attention_bwd_block(q, v, v, do, lse, delta, *a)


def _scale_squared(q, k, v, do, lse, delta, scale, *a):
    dq, dk, dv = oracle.attention_bwd_block(q, k, v, do, lse, delta, scale, *a)
    return scale * dq, scale * dk, dv


@pytest.mark.parametrize("mutant", [_delta_dropped, _lse_base2, _v_for_k, _scale_squared])
def test_block_bwd_pin_rejects_planted_mistakes(mutant):
    case = _block_bwd_case(11, True, None)
    q, k, v, do, lse, delta, q_pos, kv_pos, _ = case
    ref = oracle.attention_bwd(q, k, v, do, 0.45, True, q_pos, kv_pos, row_block=4)
    got = _sum_of_block_shares(case, True, None, block_fn=mutant)
    assert not all(np.allclose(g, w, atol=1e-12) for g, w in zip(got, ref))
