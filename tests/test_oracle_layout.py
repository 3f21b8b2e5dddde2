"""Pins for the oracle's layout functions (CPU only).

Pinned to: the rank/chunk table the Megatron CP blog prints for cp_size = 4
(tests/golden/head_tail_cp4.txt), the padding rule and the global-position
rule of the same section, and brute-force properties (bijection, inverse,
equal causal work per rank under head-tail). The striped layout is pinned to
its definition (token g on rank g mod cp) and to the closed form of its
per-rank causal work.
"""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "head_tail_cp4.txt")


def _golden_table():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append([int(x) for x in line.split()])
    return rows


def test_head_tail_table_cp4_matches_page():
    table = _golden_table()
    assert [r[0] for r in table] == [0, 1, 2, 3]
    assert oracle.rank_chunks(4, oracle.HEAD_TAIL) == [r[1:] for r in table]


@pytest.mark.parametrize("c", [1, 3, 5])
def test_head_tail_slots_follow_table_cp4(c):
    L = 8 * c
    Lp, src, pos = oracle.perm_index(L, 4, oracle.HEAD_TAIL)
    assert Lp == L
    for rank, front, tail in _golden_table():
        local = pos[rank * 2 * c:(rank + 1) * 2 * c]
        assert list(local[:c]) == list(range(front * c, (front + 1) * c))
        assert list(local[c:]) == list(range(tail * c, (tail + 1) * c))


@pytest.mark.parametrize("cp", list(range(1, 17)))
@pytest.mark.parametrize("L", [0, 1, 7, 64, 97, 256])
def test_bijection_padding_and_inverse(cp, L):
    for layout in (oracle.HEAD_TAIL, oracle.CONTIGUOUS, oracle.STRIPED):
        Lp, src, pos = oracle.perm_index(L, cp, layout)
        m = 2 * cp if layout == oracle.HEAD_TAIL else cp
        assert Lp % m == 0 and Lp >= L and Lp - L < m
        assert sorted(pos.tolist()) == list(range(Lp))          # bijection onto padded sequence
        assert np.array_equal(src[pos < L], pos[pos < L])
        assert np.all(src[pos >= L] == -1)
        rng = np.random.default_rng(cp * 1000 + L)
        x = rng.standard_normal((2, 3, L, 4))
        y, pos2 = oracle.permute(x, cp, layout)
        assert np.array_equal(pos2, pos)
        assert np.all(y[..., pos >= L, :] == 0.0)                  # pad rows are zero
        assert np.array_equal(oracle.unpermute(y, L, cp, layout), x)


@pytest.mark.parametrize("cp", [1, 2, 3, 4, 8, 16])
def test_rank_holds_chunks_r_and_mirror(cp):
    c = 5
    L = 2 * cp * c
    Lp, src, pos = oracle.perm_index(L, cp, oracle.HEAD_TAIL)
    for r in range(cp):
        local = pos[r * 2 * c:(r + 1) * 2 * c]
        chunks = sorted(set((local // c).tolist()))
        assert chunks == sorted({r, 2 * cp - 1 - r})
        # positions are global (not renumbered) and strictly increasing per chunk
        assert np.all(np.diff(local[:c]) == 1) and np.all(np.diff(local[c:]) == 1)
        # and non-decreasing across the whole local slice (front chunk precedes tail)
        assert np.all(np.diff(local) > 0)


def test_contiguous_is_identity():
    Lp, src, pos = oracle.perm_index(96, 8, oracle.CONTIGUOUS)
    assert np.array_equal(pos, np.arange(96)) and np.array_equal(src, np.arange(96))


@pytest.mark.parametrize("cp,c", [(2, 3), (3, 2), (4, 4)])
def test_head_tail_balances_causal_work(cp, c):
    L = 2 * cp * c
    counts = oracle.causal_pairs_per_rank(L, cp, oracle.HEAD_TAIL)
    assert counts == [2 * c * c * cp + c] * cp
    naive = oracle.causal_pairs_per_rank(L, cp, oracle.CONTIGUOUS)
    assert all(a < b for a, b in zip(naive, naive[1:]))          # contiguous is imbalanced
    assert sum(naive) == sum(counts) == L * (L + 1) // 2


@pytest.mark.parametrize("cp", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("L", [1, 10, 64, 97])
def test_striped_token_g_on_rank_g_mod_cp(cp, L):
    Lp, src, pos = oracle.perm_index(L, cp, oracle.STRIPED)
    n = Lp // cp
    assert Lp % cp == 0 and Lp - L < cp
    for r in range(cp):
        local = pos[r * n:(r + 1) * n]
        assert np.all(local % cp == r)
        assert local[0] == r and np.all(np.diff(local) == cp)   # increasing, stride cp


@pytest.mark.parametrize("cp,n", [(2, 3), (3, 4), (4, 5), (8, 2)])
def test_striped_causal_work_closed_form(cp, n):
    # query j*cp + r sees j*cp + r + 1 keys; summed over j = 0..n-1
    L = cp * n
    counts = oracle.causal_pairs_per_rank(L, cp, oracle.STRIPED)
    assert counts == [cp * n * (n - 1) // 2 + n * (r + 1) for r in range(cp)]
    assert sum(counts) == L * (L + 1) // 2
    naive = oracle.causal_pairs_per_rank(L, cp, oracle.CONTIGUOUS)
    assert max(counts) - min(counts) == n * (cp - 1) <= max(naive) - min(naive)


def test_striped_has_no_chunks():
    with pytest.raises(ValueError):
        oracle.rank_chunks(4, oracle.STRIPED)


def test_invalid_arguments():
    with pytest.raises(ValueError):
        oracle.padded_len(10, 0, oracle.HEAD_TAIL)
    with pytest.raises(ValueError):
        oracle.padded_len(10, 2, 7)
