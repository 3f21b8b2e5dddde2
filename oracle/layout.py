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


def varlen_index(cu_seqlens, cp, layout, align=1):
    """Layout of a pack of sequences with boundaries cu_seqlens [nseq + 1].

    Returns (Tp, src, pos, seg, gkey), each per slot of the permuted pack:
    src = index into the unpadded pack or -1 for padding, pos = position inside
    the sequence (padding continues L_i, L_i + 1, ...), seg = sequence id or -1
    for padding, gkey = offset of the sequence in the padded pack + pos.
    Rank r's slice (rows [r Tp / cp, (r + 1) Tp / cp)) holds, for every
    sequence in order, the rows rank r holds under ``perm_index`` of that
    sequence alone.

    align > 1 (a reading: the page fixes only the multiple-of-2cp padding, as
    the least a sequence needs; padding more is allowed since pad rows are
    masked) pads every sequence's share on every rank to a multiple of align
    rows, so that align-row tiles never straddle two sequences. The extra pad
    rows of rank r's share come after its real rows, with positions
    Lp_i + r * e + k (e extra rows per rank, k = 0..e-1), past every position
    the sequence uses; the sequence then occupies cp * (its aligned share) rows
    of the padded pack, which is what the next sequence's offset counts.
    """
    cu = [int(x) for x in cu_seqlens]
    if any(b < a for a, b in zip(cu, cu[1:])) or (cu and cu[0] != 0):
        raise ValueError("cu_seqlens must start at 0 and be non-decreasing")
    if align < 1:
        raise ValueError("align must be positive")
    per_rank = [[] for _ in range(cp)]
    offset = 0
    for i in range(len(cu) - 1):
        L = cu[i + 1] - cu[i]
        Lp, src_i, pos_i = perm_index(L, cp, layout)
        n = Lp // cp
        n_al = -(-n // align) * align
        e = n_al - n
        for r in range(cp):
            for j in range(r * n, (r + 1) * n):
                real = src_i[j] >= 0
                per_rank[r].append((cu[i] + src_i[j] if real else -1, pos_i[j], i if real else -1,
                                    offset + pos_i[j]))
            for kk in range(e):
                p = Lp + r * e + kk
                per_rank[r].append((-1, p, -1, offset + p))
        offset += cp * n_al
    rows = [t for r in range(cp) for t in per_rank[r]]
    Tp = len(rows)
    src = np.array([t[0] for t in rows], dtype=np.int64)
    pos = np.array([t[1] for t in rows], dtype=np.int64)
    seg = np.array([t[2] for t in rows], dtype=np.int64)
    gkey = np.array([t[3] for t in rows], dtype=np.int64)
    return Tp, src, pos, seg, gkey


def varlen_permute(x, cu_seqlens, cp, layout, align=1):
    """x [..., T, D] (a pack) -> y [..., Tp, D] in rank-major order; pad rows zero."""
    Tp, src, _, _, _ = varlen_index(cu_seqlens, cp, layout, align)
    y = np.zeros(x.shape[:-2] + (Tp, x.shape[-1]), dtype=x.dtype)
    for i in range(Tp):
        if src[i] >= 0:
            y[..., i, :] = x[..., src[i], :]
    return y


def varlen_unpermute(y, cu_seqlens, cp, layout, align=1):
    """Inverse of varlen_permute: y [..., Tp, D] -> x [..., T, D], pad rows dropped."""
    Tp, src, _, _, _ = varlen_index(cu_seqlens, cp, layout, align)
    T = int(cu_seqlens[-1])
    x = np.zeros(y.shape[:-2] + (T, y.shape[-1]), dtype=y.dtype)
    for i in range(Tp):
        if src[i] >= 0:
            x[..., src[i], :] = y[..., i, :]
    return x
