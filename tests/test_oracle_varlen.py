"""Pins for the oracle's packed-sequence (varlen) layout and segment masks (CPU).

Pinned to: the single-sequence layout (a pack of one sequence is exactly the
plain layout), per-sequence rank shares (every sequence is laid out on its own,
[Megatron-CP] "Symmetric chunk assignment" applied per sequence), bijection and
inverse, and -- independently of the masking code -- packed attention equal to
the concatenation of per-sequence attention (forward and gradient), also through
the emulated ring over the permuted pack.
"""
import numpy as np
import pytest

import oracle

PACKS = [[0, 5, 16, 16, 23], [0, 64], [0, 1, 2, 3], [0, 30, 33, 100]]
LAYOUTS = [oracle.HEAD_TAIL, oracle.STRIPED, oracle.CONTIGUOUS]


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("cp", [1, 2, 4])
def test_single_sequence_is_the_plain_layout(layout, cp):
    for L in (1, 29, 64):
        Tp, src, pos, seg, gkey = oracle.varlen_index([0, L], cp, layout)
        Lp, src1, pos1 = oracle.perm_index(L, cp, layout)
        assert Tp == Lp and np.array_equal(src, src1) and np.array_equal(pos, pos1)
        assert np.array_equal(gkey, pos1)
        assert np.array_equal(seg, np.where(src1 >= 0, 0, -1))


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("cp", [1, 2, 3, 4])
@pytest.mark.parametrize("cu", PACKS)
def test_every_sequence_laid_out_on_its_own(layout, cp, cu):
    Tp, src, pos, seg, gkey = oracle.varlen_index(cu, cp, layout)
    n = Tp // cp
    assert Tp % cp == 0
    for r in range(cp):
        sl = slice(r * n, (r + 1) * n)
        off = 0
        for i in range(len(cu) - 1):
            L = cu[i + 1] - cu[i]
            Lp, s1, p1 = oracle.perm_index(L, cp, layout)
            m = Lp // cp
            part_src = src[sl][off:off + m]
            part_pos = pos[sl][off:off + m]
            exp_src = np.where(s1[r * m:(r + 1) * m] >= 0, s1[r * m:(r + 1) * m] + cu[i], -1)
            assert np.array_equal(part_src, exp_src)
            assert np.array_equal(part_pos, p1[r * m:(r + 1) * m])
            assert np.all(seg[sl][off:off + m] == np.where(exp_src >= 0, i, -1))
            off += m
        assert off == n
        assert np.all(np.diff(gkey[sl]) > 0)          # increasing along every rank slice


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("cu", PACKS)
def test_bijection_and_inverse(layout, cu):
    Tp, src, pos, seg, gkey = oracle.varlen_index(cu, 3, layout)
    T = cu[-1]
    assert sorted(src[src >= 0].tolist()) == list(range(T))
    x = np.random.default_rng(1).standard_normal((2, T, 3))
    y = oracle.varlen_permute(x, cu, 3, layout)
    assert np.all(y[:, src < 0] == 0)
    assert np.array_equal(oracle.varlen_unpermute(y, cu, 3, layout), x)


def _per_sequence(fn, cu, *arrays):
    outs = [fn(*[a[..., cu[i]:cu[i + 1], :] for a in arrays]) for i in range(len(cu) - 1)]
    return outs


@pytest.mark.parametrize("causal", [True, False])
def test_packed_attention_is_per_sequence_attention(causal):
    cu = [0, 7, 20, 21, 40]
    rng = np.random.default_rng(2)
    q, k, v, do = (rng.standard_normal((2, cu[-1], 8)) for _ in range(4))
    tok_seg = np.concatenate([np.full(cu[i + 1] - cu[i], i) for i in range(len(cu) - 1)])
    tok_pos = np.concatenate([np.arange(cu[i + 1] - cu[i]) for i in range(len(cu) - 1)])
    o, lse = oracle.attention(q, k, v, 0.4, causal, tok_pos, tok_pos, q_seg=tok_seg, kv_seg=tok_seg, row_block=6)
    grads = oracle.attention_bwd(q, k, v, do, 0.4, causal, tok_pos, tok_pos, q_seg=tok_seg, kv_seg=tok_seg,
                                 row_block=6)
    for i in range(len(cu) - 1):
        sl = slice(cu[i], cu[i + 1])
        oi, li = oracle.attention(q[:, sl], k[:, sl], v[:, sl], 0.4, causal)
        np.testing.assert_allclose(o[:, sl], oi, atol=1e-12)
        np.testing.assert_allclose(lse[:, sl], li, atol=1e-12)
        gi = oracle.attention_bwd(q[:, sl], k[:, sl], v[:, sl], do[:, sl], 0.4, causal)
        for g, r in zip(grads, gi):
            np.testing.assert_allclose(g[:, sl], r, atol=1e-12)


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("cp", [1, 2, 3])
def test_ring_over_permuted_pack_is_per_sequence_attention(layout, cp):
    cu = [0, 9, 22, 23, 35]
    rng = np.random.default_rng(3)
    q, k, v = (rng.standard_normal((1, cu[-1], 4)) for _ in range(3))
    Tp, src, pos, seg, gkey = oracle.varlen_index(cu, cp, layout)
    qp, kp, vp = (oracle.varlen_permute(x, cu, cp, layout) for x in (q, k, v))
    o, lse = oracle.ring_emulate(qp, kp, vp, gkey, cp, 0.5, True, seg=seg)
    ou = oracle.varlen_unpermute(o, cu, cp, layout)
    for i in range(len(cu) - 1):
        sl = slice(cu[i], cu[i + 1])
        oi, li = oracle.attention(q[:, sl], k[:, sl], v[:, sl], 0.5, True)
        np.testing.assert_allclose(ou[:, sl], oi, atol=1e-12)
    lu = oracle.varlen_unpermute(lse[..., None], cu, cp, layout)[..., 0]
    for i in range(len(cu) - 1):
        sl = slice(cu[i], cu[i + 1])
        _, li = oracle.attention(q[:, sl], k[:, sl], v[:, sl], 0.5, True)
        np.testing.assert_allclose(lu[:, sl], li, atol=1e-12)


def test_segment_mask_planted_mistake_is_caught():
    # dropping the segment test lets queries see earlier sequences
    cu = [0, 4, 9]
    rng = np.random.default_rng(4)
    q, k, v = (rng.standard_normal((1, 9, 4)) for _ in range(3))
    o_wrong, _ = oracle.attention(q, k, v, 0.5, True, np.arange(9), np.arange(9))
    o_right, _ = oracle.attention(q[:, 4:], k[:, 4:], v[:, 4:], 0.5, True)
    assert np.max(np.abs(o_wrong[:, 4:] - o_right)) > 1e-3


def test_invalid_pack():
    with pytest.raises(ValueError):
        oracle.varlen_index([0, 5, 3], 2, oracle.HEAD_TAIL)
    with pytest.raises(ValueError):
        oracle.varlen_index([1, 5], 2, oracle.HEAD_TAIL)


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("cp", [1, 2, 3, 4])
@pytest.mark.parametrize("align", [1, 4, 8, 128])
@pytest.mark.parametrize("cu", PACKS)
def test_aligned_shares(layout, cp, align, cu):
    """With align, every sequence's share of every rank slice starts and ends
    on a multiple of align rows; its real rows are those of the unaligned
    layout, in order, followed only by pad rows; gkey still increases along
    every slice, and align = 1 is the unaligned layout."""
    Tp, src, pos, seg, gkey = oracle.varlen_index(cu, cp, layout, align)
    T1, src1, pos1, seg1, gkey1 = oracle.varlen_index(cu, cp, layout)
    if align == 1:
        assert Tp == T1 and all(np.array_equal(a, b) for a, b in ((src, src1), (pos, pos1), (seg, seg1),
                                                                  (gkey, gkey1)))
    n, n1 = Tp // cp, T1 // cp
    assert Tp % cp == 0
    for r in range(cp):
        sl, sl1 = slice(r * n, (r + 1) * n), slice(r * n1, (r + 1) * n1)
        off = off1 = 0
        for i in range(len(cu) - 1):
            m1 = oracle.padded_len(cu[i + 1] - cu[i], cp, layout) // cp
            m = -(-m1 // align) * align
            assert off % align == 0
            assert np.array_equal(src[sl][off:off + m1], src1[sl1][off1:off1 + m1])
            assert np.array_equal(pos[sl][off:off + m1], pos1[sl1][off1:off1 + m1])
            assert np.all(src[sl][off + m1:off + m] == -1) and np.all(seg[sl][off + m1:off + m] == -1)
            assert np.all(pos[sl][off + m1:off + m] >= cp * m1)   # past every position of the sequence
            off += m
            off1 += m1
        assert off == n
        assert np.all(np.diff(gkey[sl]) > 0)
    assert sorted(src[src >= 0].tolist()) == list(range(cu[-1]))


@pytest.mark.parametrize("align", [8, 128])
def test_aligned_pack_attention_is_per_sequence_attention(align):
    """The aligned layout changes only padding: attention over the permuted
    pack with its segment mask, put back in pack order, is still per-sequence
    attention (forward and gradient)."""
    cu = [0, 30, 33, 100]
    cp = 2
    rng = np.random.default_rng(11)
    q, k, v, do = (rng.standard_normal((1, 2, cu[-1], 4)) for _ in range(4))
    Tp, src, pos, seg, gkey = oracle.varlen_index(cu, cp, oracle.HEAD_TAIL, align)
    qp, kp, vp, dop = (oracle.varlen_permute(x, cu, cp, oracle.HEAD_TAIL, align) for x in (q, k, v, do))
    segk = np.where(seg >= 0, seg, -1)
    o, _ = oracle.attention(qp, kp, vp, 0.5, True, gkey, gkey, None, q_seg=seg, kv_seg=segk)
    g = oracle.attention_bwd(qp, kp, vp, dop, 0.5, True, gkey, gkey, None, q_seg=seg, kv_seg=segk)
    o_ref = np.concatenate(_per_sequence(lambda a, b, c: oracle.attention(a, b, c, 0.5, True)[0], cu, q, k, v), -2)
    np.testing.assert_allclose(oracle.varlen_unpermute(o, cu, cp, oracle.HEAD_TAIL, align), o_ref, atol=1e-12)
    g_ref = _per_sequence(lambda a, b, c, d: oracle.attention_bwd(a, b, c, d, 0.5, True), cu, q, k, v, do)
    for j in range(3):
        want = np.concatenate([x[j] for x in g_ref], -2)
        np.testing.assert_allclose(oracle.varlen_unpermute(g[j], cu, cp, oracle.HEAD_TAIL, align), want, atol=1e-12)
