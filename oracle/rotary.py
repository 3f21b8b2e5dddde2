"""Oracle: rotary position embedding at carried global positions (test
infrastructure only).

Why it is on the path: the blog "Context Parallelism v.s. Sequence
Parallelism (Megatron-LM)", section "Symmetric chunk assignment", points out
that RoPE consumes each token's position, so a rank holding chunk r and chunk
2*cp-1-r must rotate with those chunks' global positions, never with local
indices 0, 1, 2, ... The pages do not restate RoPE itself; the definition
used is the one published with it (Su et al., "RoFormer: Enhanced Transformer
with Rotary Position Embedding", 2021): the head vector is cut into D/2 pairs,
pair i is rotated in its plane by the angle p * base^(-2i/D) for a token at
position p.

Readings where the pages are silent:
  * base = 10000 unless given;
  * two pairings are supported: INTERLEAVED pairs (x[2i], x[2i+1]) as in the
    paper's formula; HALF pairs (x[i], x[i + D/2]) (the "rotate half" form
    that Megatron-LM uses by default), both with frequency index i;
  * the rotation of pair (a, b) by angle t is (a cos t - b sin t,
    a sin t + b cos t);
  * the gradient with respect to the un-rotated input is the transposed
    (inverse) rotation of the upstream gradient, since each rotation is
    orthogonal.
"""
import numpy as np

HALF = 0
INTERLEAVED = 1


def pair_index(D, style):
    """(first, second) element indices of the D/2 rotation pairs; pair i uses
    frequency index i."""
    if D % 2:
        raise ValueError("D must be even")
    i = np.arange(D // 2)
    if style == INTERLEAVED:
        return 2 * i, 2 * i + 1
    if style == HALF:
        return i, i + D // 2
    raise ValueError("unknown rope style")


def angles(pos, D, base=10000.0):
    """[len(pos), D/2] rotation angles p * base^(-2i/D) in float64."""
    pos = np.asarray(pos, dtype=np.float64)
    inv_freq = base ** (-2.0 * np.arange(D // 2, dtype=np.float64) / D)
    return pos[:, None] * inv_freq[None, :]


def _rotate(x, pos, base, style, sign):
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    a_idx, b_idx = pair_index(D, style)
    t = sign * angles(pos, D, base)             # [L, D/2], broadcast over leading dims
    c, s = np.cos(t), np.sin(t)
    a, b = x[..., a_idx], x[..., b_idx]
    y = np.empty_like(x)
    y[..., a_idx] = a * c - b * s
    y[..., b_idx] = a * s + b * c
    return y


def rope(x, pos, base=10000.0, style=HALF):
    """x [..., L, D] rotated at positions pos [L]."""
    return _rotate(x, pos, base, style, 1.0)


def rope_grad(dy, pos, base=10000.0, style=HALF):
    """Gradient with respect to the input of ``rope`` for upstream dy
    [..., L, D]: the inverse (transposed) rotation."""
    return _rotate(dy, pos, base, style, -1.0)
