"""Oracle: context-parallel sequence layouts (test infrastructure only).

Follows the blog "Context Parallelism v.s. Sequence Parallelism (Megatron-LM)",
section "Symmetric chunk assignment":
  * the sequence is cut into 2*cp_size equal chunks;
  * rank r holds chunk r followed by chunk 2*cp_size-1-r (the page's table for
    cp_size=4: rank 0 <- chunks 0,7; rank 1 <- 1,6; rank 2 <- 2,5; rank 3 <- 3,4);
  * every token keeps its global position id (no renumbering 0,1,2,... per rank);
  * the length must be padded to a multiple of 2*cp_size or the layout breaks.
The contiguous ("naive") layout is the left half of that section's figure
caption: rank r holds the r-th of cp_size contiguous pieces.

The striped layout follows the page "Sequence parallelism and ring attention"
(aiunderstanding.org), section on the future of sequence parallelism, which
names striped attention as a variant that rebalances the causal work; the
reading taken is the published Striped Attention assignment (Brandon et al.,
2023): token g goes to rank g mod cp_size, each rank keeping its tokens in
increasing order, and the length is padded to a multiple of cp_size.

Readings where the page is silent: padding goes at the tail of the global
sequence, pad slots carry the positions L, L+1, ... they would have in the
padded sequence, and pad values are zero. Ranks are concatenated in rank order.
"""
import numpy as np

CONTIGUOUS = 0
HEAD_TAIL = 1
STRIPED = 2


def _n_chunks(cp, layout):
    if cp < 1:
        raise ValueError("cp_size must be >= 1")
    if layout == HEAD_TAIL:
        return 2 * cp
    if layout in (CONTIGUOUS, STRIPED):
        return cp
    raise ValueError("unknown layout")


def padded_len(L, cp, layout):
    """Smallest Lp >= L that splits into equal chunks (2*cp of them for
    head-tail, cp for contiguous; striped needs the same cp equal shares)."""
    n = _n_chunks(cp, layout)
    if L < 0:
        raise ValueError("L must be >= 0")
    return -(-L // n) * n


def rank_chunks(cp, layout):
    """List, per rank, of the global chunk indices it holds, in local order
    (chunked layouts only)."""
    if layout == STRIPED:
        raise ValueError("the striped layout is not made of chunks")
    if layout == HEAD_TAIL:
        return [[r, 2 * cp - 1 - r] for r in range(cp)]
    _n_chunks(cp, layout)
    return [[r] for r in range(cp)]


def perm_index(L, cp, layout):
    """Return (Lp, src, pos) for the permuted (rank-major) sequence.

    Slot i of the permuted sequence holds global token pos[i]; src[i] is the
    index in the unpadded input it copies, or -1 for a pad slot.
    """
    Lp = padded_len(L, cp, layout)
    n = _n_chunks(cp, layout)
    c = Lp // n
    if layout == STRIPED:
        # rank r's tokens are r, r + cp, r + 2 cp, ... (c = Lp / cp of them)
        pos = np.array([j * cp + r for r in range(cp) for j in range(c)], dtype=np.int64)
        src = np.where(pos < L, pos, -1)
        return Lp, src, pos
    chunks = [np.arange(k * c, (k + 1) * c, dtype=np.int64) for k in range(n)]
    pieces = [chunks[k] for owned in rank_chunks(cp, layout) for k in owned]
    pos = np.concatenate(pieces) if pieces else np.zeros(0, np.int64)
    src = np.where(pos < L, pos, -1)
    return Lp, src, pos


def permute(x, cp, layout):
    """x [..., L, D] -> (y [..., Lp, D], pos [Lp]); pad rows are zero."""
    L = x.shape[-2]
    Lp, src, pos = perm_index(L, cp, layout)
    y = np.zeros(x.shape[:-2] + (Lp, x.shape[-1]), dtype=x.dtype)
    for i in range(Lp):
        if src[i] >= 0:
            y[..., i, :] = x[..., src[i], :]
    return y, pos


def unpermute(y, L, cp, layout):
    """Inverse of permute: y [..., Lp, D] -> x [..., L, D], pad rows dropped."""
    Lp, src, _ = perm_index(L, cp, layout)
    if y.shape[-2] != Lp:
        raise ValueError("y has the wrong padded length")
    x = np.zeros(y.shape[:-2] + (L, y.shape[-1]), dtype=y.dtype)
    for i in range(Lp):
        if src[i] >= 0:
            x[..., src[i], :] = y[..., i, :]
    return x
