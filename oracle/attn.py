"""Oracle: softmax attention, the online-softmax fold, the emulated ring, and
the attention gradient, all in float64 (test infrastructure only).

What the method reaches exactly (up to rounding order) is plain full-sequence
softmax attention: the Ultralytics glossary "Context Parallelism", section
"How context parallelism works", states the ring result equals full-sequence
attention apart from ordinary numerical differences, and the aiunderstanding.org
page "Sequence parallelism and ring attention", section "Technical insight",
says the blockwise online-softmax result is mathematically identical to full
attention. So ``attention`` below is that definition written out; ``merge`` and
``ring_emulate`` restate the blockwise algorithm of that page (local Q fixed,
K/V blocks arriving hop by hop, each partial folded into the accumulator with
a running max / normaliser) and are used only to check invariants.

Conventions (readings where the pages are silent):
  * scale multiplies Q K^T before the softmax;
  * a key is visible to a query iff (not causal or kv_pos <= q_pos) and
    (kv_valid is None or kv_pos < kv_valid);
  * LSE is the natural-log normaliser log(sum_j exp(scale * q.k_j)) over the
    visible keys; a row with no visible key has LSE = -inf and O = 0.
"""
import numpy as np


def visible_mask(q_pos, kv_pos, causal, kv_valid=None, q_seg=None, kv_seg=None):
    """Boolean [Lq, Lk] matrix of visible (query, key) pairs. With segment ids
    (packed sequences) a key is visible only to queries of its own segment,
    and a key whose segment id is negative (padding) to none."""
    q_pos = np.asarray(q_pos, dtype=np.int64)
    kv_pos = np.asarray(kv_pos, dtype=np.int64)
    m = np.ones((q_pos.shape[0], kv_pos.shape[0]), dtype=bool)
    if causal:
        m &= kv_pos[None, :] <= q_pos[:, None]
    if kv_valid is not None:
        m &= kv_pos[None, :] < kv_valid
    if kv_seg is not None:
        q_seg = np.asarray(q_seg, dtype=np.int64)
        kv_seg = np.asarray(kv_seg, dtype=np.int64)
        m &= (kv_seg[None, :] == q_seg[:, None]) & (kv_seg[None, :] >= 0)
    return m


def _default_pos(n):
    return np.arange(n, dtype=np.int64)


def _attention_2d(q, k, v, scale, mask):
    """One (batch, head): q [Lq, D], k/v [Lk, D], mask [Lq, Lk] -> O, LSE."""
    s = scale * (q @ k.T)
    s = np.where(mask, s, -np.inf)
    m = s.max(axis=1, initial=-np.inf)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    p = np.exp(s - m_safe[:, None])            # exp(-inf) = 0 on masked entries
    l = p.sum(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        lse = np.where(finite, m_safe + np.log(l), -np.inf)
        o = np.where(finite[:, None], (p @ v) / np.where(finite, l, 1.0)[:, None], 0.0)
    return o, lse


def attention(q, k, v, scale, causal, q_pos=None, kv_pos=None, kv_valid=None, row_block=256, q_seg=None,
              kv_seg=None):
    """Full softmax attention in float64.

    q [..., Lq, D], k/v [..., Lk, D] (any float dtype; computed in float64 from
    the exact values given). Returns O [..., Lq, D] and LSE [..., Lq].
    Query rows are evaluated in independent blocks of ``row_block`` rows.
    Optional segment ids restrict every query to the keys of its own segment
    (packed sequences).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    Lq, D = q.shape[-2], q.shape[-1]
    Lk = k.shape[-2]
    q_pos = _default_pos(Lq) if q_pos is None else np.asarray(q_pos, dtype=np.int64)
    kv_pos = _default_pos(Lk) if kv_pos is None else np.asarray(kv_pos, dtype=np.int64)
    lead = q.shape[:-2]
    nb = int(np.prod(lead, dtype=np.int64))
    qf = q.reshape(nb, Lq, D)
    kf = k.reshape(nb, Lk, D)
    vf = v.reshape(nb, Lk, v.shape[-1])
    o = np.zeros((qf.shape[0], Lq, vf.shape[-1]))
    lse = np.zeros((qf.shape[0], Lq))
    for b in range(qf.shape[0]):
        for r0 in range(0, Lq, row_block):
            r1 = min(Lq, r0 + row_block)
            mask = visible_mask(q_pos[r0:r1], kv_pos, causal, kv_valid,
                                None if q_seg is None else np.asarray(q_seg)[r0:r1], kv_seg)
            o[b, r0:r1], lse[b, r0:r1] = _attention_2d(qf[b, r0:r1], kf[b], vf[b], scale, mask)
    return o.reshape(lead + (Lq, vf.shape[-1])), lse.reshape(lead + (Lq,))


def merge(o_acc, lse_acc, o_blk, lse_blk):
    """Online-softmax fold of two partial results over disjoint key sets.

    LSE' = log(exp(LSE_acc) + exp(LSE_blk)), computed around the larger of the
    two; O' = exp(LSE_acc - LSE') O_acc + exp(LSE_blk - LSE') O_blk.
    A side with LSE = -inf contributes nothing; both -inf gives -inf and O = 0.
    """
    o_acc = np.asarray(o_acc, dtype=np.float64)
    o_blk = np.asarray(o_blk, dtype=np.float64)
    a = np.asarray(lse_acc, dtype=np.float64)
    b = np.asarray(lse_blk, dtype=np.float64)
    m = np.maximum(a, b)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    wa = np.exp(a - m_safe)
    wb = np.exp(b - m_safe)
    tot = wa + wb
    with np.errstate(divide="ignore", invalid="ignore"):
        lse = np.where(finite, m_safe + np.log(np.where(finite, tot, 1.0)), -np.inf)
        ca = np.where(finite, wa / np.where(finite, tot, 1.0), 0.0)
        cb = np.where(finite, wb / np.where(finite, tot, 1.0), 0.0)
    o = ca[..., None] * o_acc + cb[..., None] * o_blk
    return o, lse


def blockwise_attention(q, k, v, scale, causal, key_blocks, q_pos=None, kv_pos=None, kv_valid=None):
    """Attention computed as partials over the given key index blocks, folded
    with ``merge`` in the given order (the blockwise scheme of the ring)."""
    Lq, Lk = q.shape[-2], k.shape[-2]
    q_pos = _default_pos(Lq) if q_pos is None else np.asarray(q_pos, dtype=np.int64)
    kv_pos = _default_pos(Lk) if kv_pos is None else np.asarray(kv_pos, dtype=np.int64)
    o = np.zeros(q.shape[:-1] + (v.shape[-1],))
    lse = np.full(q.shape[:-1], -np.inf)
    for idx in key_blocks:
        idx = np.asarray(idx, dtype=np.int64)
        ob, lb = attention(q, k[..., idx, :], v[..., idx, :], scale, causal,
                           q_pos=q_pos, kv_pos=kv_pos[idx], kv_valid=kv_valid)
        o, lse = merge(o, lse, ob, lb)
    return o, lse


def ring_emulate(q, k, v, pos, cp, scale, causal, kv_valid=None, seg=None):
    """The ring of the pages, emulated: q/k/v [..., Lp, D] in permuted
    (rank-major) order with positions ``pos``. Rank r keeps its local Q fixed;
    at hop t it holds the K/V block of rank s = (r - t) mod cp (blocks move to
    the next device each hop) and folds that block's partial attention into its
    accumulator. Returns O, LSE in the same permuted order."""
    Lp = q.shape[-2]
    if Lp % cp:
        raise ValueError("Lp must be a multiple of cp")
    n = Lp // cp
    pos = np.asarray(pos, dtype=np.int64)
    o = np.zeros(q.shape[:-1] + (v.shape[-1],))
    lse = np.full(q.shape[:-1], -np.inf)
    for r in range(cp):
        rows = slice(r * n, (r + 1) * n)
        o_acc = np.zeros(q[..., rows, :].shape[:-1] + (v.shape[-1],))
        lse_acc = np.full(q[..., rows, :].shape[:-1], -np.inf)
        for t in range(cp):
            s = (r - t) % cp
            keys = slice(s * n, (s + 1) * n)
            ob, lb = attention(q[..., rows, :], k[..., keys, :], v[..., keys, :], scale, causal,
                               q_pos=pos[rows], kv_pos=pos[keys], kv_valid=kv_valid,
                               q_seg=None if seg is None else seg[rows], kv_seg=None if seg is None else seg[keys])
            o_acc, lse_acc = merge(o_acc, lse_acc, ob, lb)
        o[..., rows, :] = o_acc
        lse[..., rows] = lse_acc
    return o, lse


def attention_bwd(q, k, v, do, scale, causal, q_pos=None, kv_pos=None, kv_valid=None, row_block=256, q_seg=None,
                  kv_seg=None):
    """Gradient of O = softmax(scale Q K^T) V (masked) for upstream dO, float64.

    Textbook softmax-attention gradient (the pages only call ``.backward()``):
      P = softmax(S), dV = P^T dO, dP = dO V^T,
      dS_ij = P_ij (dP_ij - sum_k P_ik dP_ik),
      dQ = scale dS K, dK = scale dS^T Q.
    Returns dq, dk, dv with the shapes of q, k, v.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    Lq, D = q.shape[-2], q.shape[-1]
    Lk = k.shape[-2]
    q_pos = _default_pos(Lq) if q_pos is None else np.asarray(q_pos, dtype=np.int64)
    kv_pos = _default_pos(Lk) if kv_pos is None else np.asarray(kv_pos, dtype=np.int64)
    nb = int(np.prod(q.shape[:-2], dtype=np.int64))
    qf, kf, vf, dof = (t.reshape(nb, t.shape[-2], t.shape[-1]) for t in (q, k, v, do))
    dq = np.zeros_like(qf)
    dk = np.zeros_like(kf)
    dv = np.zeros_like(vf)
    for b in range(qf.shape[0]):
        for r0 in range(0, Lq, row_block):
            r1 = min(Lq, r0 + row_block)
            mask = visible_mask(q_pos[r0:r1], kv_pos, causal, kv_valid,
                                None if q_seg is None else np.asarray(q_seg)[r0:r1], kv_seg)
            s = np.where(mask, scale * (qf[b, r0:r1] @ kf[b].T), -np.inf)
            m = s.max(axis=1, initial=-np.inf)
            m_safe = np.where(np.isfinite(m), m, 0.0)
            e = np.exp(s - m_safe[:, None])
            l = e.sum(axis=1)
            p = e / np.where(l > 0, l, 1.0)[:, None]
            dv[b] += p.T @ dof[b, r0:r1]
            dp = dof[b, r0:r1] @ vf[b].T
            ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
            dq[b, r0:r1] = scale * (ds @ kf[b])
            dk[b] += scale * (ds.T @ qf[b, r0:r1])
    return dq.reshape(q.shape), dk.reshape(k.shape), dv.reshape(v.shape)


def attention_bwd_block(q, k, v, do, lse, delta, scale, causal, q_pos=None, kv_pos=None, kv_valid=None):
    """One key block's share of the attention gradient, float64: what a rank
    computes at one hop of the ring backward, where the softmax of a query row
    spans every block but only this one is at hand. The row's final LSE and
    delta_i = sum_d dO_id O_id (O the final output) stand in for the rest:
      P_ij = exp(scale q_i.k_j - LSE_i) on visible pairs, 0 elsewhere,
      dV = P^T dO, dP = dO V^T, dS_ij = P_ij (dP_ij - delta_i),
      dQ = scale dS K (this block's part), dK = scale dS^T Q, dV as above.
    Since sum_j P_ij dP_ij = sum_d dO_id O_id, the shares summed over a
    partition of the keys are ``attention_bwd``. lse [..., Lq], delta
    [..., Lq]; returns dq [..., Lq, D], dk, dv [..., Lk, D]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    delta = np.asarray(delta, dtype=np.float64)
    Lq, Lk = q.shape[-2], k.shape[-2]
    q_pos = _default_pos(Lq) if q_pos is None else np.asarray(q_pos, dtype=np.int64)
    kv_pos = _default_pos(Lk) if kv_pos is None else np.asarray(kv_pos, dtype=np.int64)
    mask = visible_mask(q_pos, kv_pos, causal, kv_valid)
    s = scale * np.einsum("...id,...jd->...ij", q, k)
    with np.errstate(over="ignore", invalid="ignore"):
        p = np.where(mask, np.exp(s - lse[..., :, None]), 0.0)
    dv = np.einsum("...ij,...id->...jd", p, do)
    dp = np.einsum("...id,...jd->...ij", do, v)
    ds = p * (dp - delta[..., :, None])
    dq = scale * np.einsum("...ij,...jd->...id", ds, k)
    dk = scale * np.einsum("...ij,...id->...jd", ds, q)
    return dq, dk, dv


def causal_pairs_per_rank(L, cp, layout):
    """Brute-force count of visible causal (query, key) pairs per rank.

    Rank r's queries are the global positions in the chunks it holds; each
    query at position p sees the keys at positions 0..p of the (unpadded)
    sequence. The head-tail assignment exists to make these counts equal
    (blog "Context Parallelism v.s. Sequence Parallelism (Megatron-LM)",
    section "Symmetric chunk assignment").
    """
    from .layout import perm_index  # local import keeps this module self-contained
    Lp, src, pos = perm_index(L, cp, layout)
    n = Lp // cp
    counts = []
    for r in range(cp):
        tot = 0
        for p in pos[r * n:(r + 1) * n]:
            if p < L:
                tot += sum(1 for key in range(L) if key <= p)
        counts.append(tot)
    return counts



def gqa_expand(x, H):
    """Grouped key/value heads seen by the query heads: x [B, H_kv, L, D] ->
    [B, H, L, D], query head h reading key/value head h // (H / H_kv).

    The blog "Context Parallelism v.s. Sequence Parallelism (Megatron-LM)",
    section "CP vs SP", sizes the ring's traffic by H_kv, the number of
    key/value heads, which is below H under grouped-query attention (GQA,
    Ainslie et al., 2023: query heads split into H_kv equal groups, each group
    sharing one key/value head). Reading: groups are contiguous runs of query
    heads."""
    x = np.asarray(x)
    H_kv = x.shape[-3]
    if H_kv < 1 or H % H_kv:
        raise ValueError("H must be a positive multiple of H_kv")
    return np.repeat(x, H // H_kv, axis=-3)


def gqa_reduce(dx, H_kv):
    """Gradient of ``gqa_expand``: [B, H, L, D] -> [B, H_kv, L, D], summing
    the gradients of the query heads of each group."""
    dx = np.asarray(dx, dtype=np.float64)
    H = dx.shape[-3]
    if H_kv < 1 or H % H_kv:
        raise ValueError("H must be a positive multiple of H_kv")
    g = H // H_kv
    return dx.reshape(dx.shape[:-3] + (H_kv, g) + dx.shape[-2:]).sum(axis=-3)
