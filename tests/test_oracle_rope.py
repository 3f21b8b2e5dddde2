"""Pins for the oracle's rotary position embedding (CPU only).

Pinned to what RoFormer's definition fixes, independently of the oracle's own
real-arithmetic formula: the complex-number form (pair = complex number,
rotation = multiplication by exp(i * angle)), the relative-position property
(q.k after rotation depends only on the position difference), the rotation
angle of every frequency at position 1, position 0 = identity, norm
preservation, the D = 2 closed form, and the gradient by central differences.
Planted mistakes (sign, frequency exponent, pairing) are each rejected.
"""
import math

import numpy as np
import pytest

import oracle
from oracle.rotary import angles, pair_index

STYLES = [oracle.ROPE_HALF, oracle.ROPE_INTERLEAVED]


def _as_complex(x, style):
    D = x.shape[-1]
    if style == oracle.ROPE_INTERLEAVED:
        return x[..., 0::2] + 1j * x[..., 1::2]
    return x[..., :D // 2] + 1j * x[..., D // 2:]


@pytest.mark.parametrize("style", STYLES)
@pytest.mark.parametrize("base", [10000.0, 500000.0])
def test_complex_multiplication_form(style, base):
    rng = np.random.default_rng(1)
    L, D = 37, 16
    x = rng.standard_normal((2, L, D))
    pos = rng.integers(0, 1 << 20, L)
    y = oracle.rope(x, pos, base, style)
    theta = np.array([base ** (-2.0 * i / D) for i in range(D // 2)])
    z = _as_complex(x, style) * np.exp(1j * pos[:, None] * theta[None, :])
    np.testing.assert_allclose(_as_complex(y, style), z, rtol=0, atol=1e-9)


@pytest.mark.parametrize("style", STYLES)
def test_relative_position_property(style):
    rng = np.random.default_rng(2)
    D = 32
    q, k = rng.standard_normal((2, 1, D))
    for m, n, s in [(5, 3, 100), (1000, 17, 77777), (0, 9, 4096)]:
        a = oracle.rope(q, [m], style=style) @ oracle.rope(k, [n], style=style).T
        b = oracle.rope(q, [m + s], style=style) @ oracle.rope(k, [n + s], style=style).T
        assert abs(a.item() - b.item()) < 1e-9
        # and it is q . R(n - m) k: rotating only the key by the difference gives the same score
        c = q @ oracle.rope(k, [n - m], style=style).T
        assert abs(a.item() - c.item()) < 1e-9


@pytest.mark.parametrize("style", STYLES)
def test_angle_of_each_frequency_at_position_one(style):
    D = 8
    first, second = pair_index(D, style)
    for i in range(D // 2):
        e = np.zeros((1, D))
        e[0, first[i]] = 1.0
        y = oracle.rope(e, [1], style=style)
        ang = math.atan2(y[0, second[i]], y[0, first[i]])
        assert abs(ang - 10000.0 ** (-2.0 * i / D)) < 1e-12
        # nothing leaks into other coordinates
        other = np.delete(y[0], [first[i], second[i]])
        assert np.all(other == 0.0)


@pytest.mark.parametrize("style", STYLES)
def test_position_zero_is_identity_and_norms_are_kept(style):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((3, 5, 64))
    assert np.array_equal(oracle.rope(x, np.zeros(5, int), style=style), x)
    pos = np.array([1, 10, 1000, 65535, 1048575])
    y = oracle.rope(x, pos, style=style)
    zx, zy = _as_complex(x, style), _as_complex(y, style)
    np.testing.assert_allclose(np.abs(zy), np.abs(zx), rtol=1e-13)


def test_d2_closed_form():
    # D = 2: one pair, frequency 1, so the pair turns by p radians
    for style in STYLES:
        for p in (0, 1, 2, 7, 123456):
            y = oracle.rope(np.array([[1.0, 0.0]]), [p], style=style)
            np.testing.assert_allclose(y[0], [math.cos(p), math.sin(p)], atol=1e-12)


@pytest.mark.parametrize("style", STYLES)
def test_gradient_by_central_differences(style):
    rng = np.random.default_rng(4)
    L, D = 4, 8
    x = rng.standard_normal((L, D))
    w = rng.standard_normal((L, D))
    pos = np.array([3, 0, 4000, 77])
    g = oracle.rope_grad(w, pos, style=style)
    h = 1e-6
    for i in range(L):
        for d in range(D):
            xp, xm = x.copy(), x.copy()
            xp[i, d] += h
            xm[i, d] -= h
            fd = (np.sum(w * oracle.rope(xp, pos, style=style)) - np.sum(w * oracle.rope(xm, pos, style=style))) / (2 * h)
            assert abs(fd - g[i, d]) < 1e-7
    np.testing.assert_allclose(oracle.rope_grad(oracle.rope(x, pos, style=style), pos, style=style), x, atol=1e-12)


def test_half_is_interleaved_on_reordered_coordinates():
    rng = np.random.default_rng(5)
    D = 16
    x = rng.standard_normal((6, D))
    pos = np.arange(6) * 1000
    # coordinate order that puts (i, i + D/2) next to each other
    order = np.stack([np.arange(D // 2), np.arange(D // 2) + D // 2], axis=1).reshape(-1)
    y_half = oracle.rope(x, pos, style=oracle.ROPE_HALF)
    y_int = oracle.rope(x[:, order], pos, style=oracle.ROPE_INTERLEAVED)
    np.testing.assert_allclose(y_half[:, order], y_int, atol=1e-12)


def _mutant(kind):
    """A RoPE with one planted mistake, built on the oracle's helpers."""
    def f(x, pos, style=oracle.ROPE_HALF):
        x = np.asarray(x, dtype=np.float64)
        D = x.shape[-1]
        a_idx, b_idx = pair_index(D, style)
        if kind == "exponent":
            t = np.asarray(pos, float)[:, None] * 10000.0 ** (-np.arange(D // 2) / D)[None, :]
        else:
            t = angles(pos, D)
        c, s = np.cos(t), np.sin(t)
        a, b = x[..., a_idx], x[..., b_idx]
        y = np.empty_like(x)
        y[..., a_idx] = a * c - b * s
        y[..., b_idx] = (-a * s + b * c) if kind == "sign" else (a * s + b * c)
        if kind == "pairing":
            y = y[..., ::-1].copy()
        return y
    return f


@pytest.mark.parametrize("kind", ["sign", "exponent", "pairing"])
def test_planted_mistakes_are_rejected(kind):
    rng = np.random.default_rng(6)
    L, D = 9, 16
    x = rng.standard_normal((L, D))
    pos = rng.integers(0, 100000, L)
    theta = np.array([10000.0 ** (-2.0 * i / D) for i in range(D // 2)])
    z = _as_complex(x, oracle.ROPE_HALF) * np.exp(1j * pos[:, None] * theta[None, :])
    bad = _mutant(kind)(x, pos)
    assert np.max(np.abs(_as_complex(bad, oracle.ROPE_HALF) - z)) > 1e-3
