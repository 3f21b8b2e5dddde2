"""Ring attention with one context-parallel rank per process.

The library's ring calls run every CP rank on one GPU. This module runs the
same ring across processes, one rank per process (one GPU each), with
``torch.distributed`` for the exchange. Each process holds its rank's slice of
the permuted sequence: rows [r L_loc, (r+1) L_loc) of what
``cp_layout_permute`` writes for Q, K and V, and the same rows of the position
array.

Sources, cited by page title and section:
  [CP-glossary]  Ultralytics glossary "Context Parallelism", section "How
                 context parallelism works": devices exchange key/value blocks;
                 in ring attention each computes a partial attention on the
                 block it holds, hands the block to the next device and repeats
                 until the whole sequence has been seen. Section "Why context
                 parallelism matters": the K/V transfer is overlapped with the
                 computation.
  [Megatron-CP]  Blog "Context Parallelism v.s. Sequence Parallelism
                 (Megatron-LM)", section "CP vs SP", communication: K and V move
                 ring-style by point-to-point sends, or by an all-gather; the
                 traffic grows as O(L H_kv).
  [Ring-page]    aiunderstanding.org "Sequence parallelism and ring attention",
                 section "Technical insight": only K/V travel, one block at a
                 time; each block's partial result is folded with the online
                 softmax (running max and normaliser).

Schedules (rank r of cp ranks; next = r+1, prev = r-1, mod cp):

  ring_fwd      hop t = 0..cp-1: rank r holds the K/V block (and positions)
                of rank s = (r - t) mod cp. It posts the send of that block to
                next and the receive of the following one from prev, computes
                the partial attention of its queries on the block in hand and
                folds it into (O, LSE), then waits for the exchange. The
                transfer for hop t+1 thus runs under hop t's arithmetic (with
                NCCL, on the communicator's stream).
  ring_bwd      (reading: the pages show only a call to ``.backward()``, so
                this is the plain gradient of the forward's fold, hop by hop.)
                delta = rowsum(dO * O) once; at hop t rank r adds block s's
                share to dQ and writes its share of dK_s, dV_s into fp32
                buffers of its own (two pairs, used in turn). Meanwhile the
                running sums of dK_s, dV_s arrive from prev, which worked on
                block s at hop t-1. They are folded in and the totals go on
                to next. After the last hop each block's sums arrive at the
                block's owner.
  allgather_fwd / allgather_bwd
                the all-gather option of [Megatron-CP]: K, V and positions are
                gathered once (the local block's arithmetic runs while the
                gather is in flight); the blocks are then folded in the same
                order as the ring, so the forward results are bit-identical to
                ``ring_fwd``. The backward of a gather is a reduce-scatter:
                every rank computes its share of dK, dV for all blocks, and
                ``reduce_scatter_tensor`` returns the sum for its own block.

Block arithmetic. By default (``KernelOps``) every block runs on this library's
kernels: ``rattn_partial_fwd`` and ``rattn_merge`` in the forward (O and LSE
come back in fp32, the fold's accumulator); ``rattn_bwd_prep`` (Delta and the
zeroed fp32 dQ accumulator), ``rattn_partial_bwd`` (one block's dQ added in
place, its dK, dV shares in fp32) and ``rattn_grad_fold`` (running sums) in
the backward. The schedules take an ``ops`` object with the same methods; their
tests on CPU (gloo ranks) pass the fp64 reference arithmetic there. Only
tensors and the exchange are handled here: no attention arithmetic lives in
this module.

With NCCL, set each process's device (``torch.cuda.set_device``) before the
first call: batched point-to-point operations need it, and every rank of the
group takes part in each exchange (all ranks call the same schedule with the
same cp, shapes and dtypes).

Failure handling. Every exchange is a ``torch.distributed`` call on the
caller's process group; give the group a short timeout so that a rank that
stops answering ends the others' next exchange with an error rather than a
hang. A rank that leaves between steps tells the others through the group's
key-value store (``RingMembership``); they check before their next step.
"""
import torch
import torch.distributed as dist

_TAG_KV = 11
_TAG_DKV = 12


class PeerLeftError(RuntimeError):
    """A rank of the ring has announced that it left."""

    def __init__(self, ranks):
        super().__init__(f"ring ranks {sorted(ranks)} have left; no further exchange is possible")
        self.ranks = sorted(ranks)


class RingMembership:
    """Host-side notice of ranks that leave between steps.

    ``store`` is a ``torch.distributed`` key-value store shared by the ranks,
    for example the ``TCPStore`` the process group was created with. A rank
    that stops calls ``leave()`` before it exits. The others call ``check()``
    before each step; it raises ``PeerLeftError`` naming every rank that left,
    before any exchange of that step is posted."""

    def __init__(self, store, rank, world_size, prefix="rattn_ring"):
        self.store = store
        self.rank = int(rank)
        self.world_size = int(world_size)
        self.prefix = prefix

    def _key(self, r):
        return f"{self.prefix}/left/{r}"

    def leave(self):
        self.store.set(self._key(self.rank), "1")

    def check(self):
        gone = [r for r in range(self.world_size) if r != self.rank and self.store.check([self._key(r)])]
        if gone:
            raise PeerLeftError(gone)


class KernelOps:
    """Block arithmetic on this library's CUDA kernels (contiguous CUDA
    tensors only; the library must be built: importing its binding raises
    otherwise, and there is no other implementation).

    fwd(q, k, v, q_pos, kv_pos, scale, causal, kv_valid) -> (o, lse)
    merge(o_acc, lse_acc, o_blk, lse_blk) -> (o_acc, lse_acc), in place
    prep(o, do) -> (delta, dq_acc): Delta and a zeroed fp32 dQ accumulator
    bwd(q, k, v, do, lse, delta, q_pos, kv_pos, scale, causal, kv_valid,
        dq_acc, dk=None, dv=None) -> (dk, dv): adds the block's dQ share to
        dq_acc; writes its dK, dV shares into dk, dv (new when None)
    fold(acc, blk) -> acc: acc += blk, in place"""

    def __init__(self):
        from . import rattn
        self._r = rattn

    def fwd(self, q, k, v, q_pos, kv_pos, scale, causal, kv_valid):
        return self._r.rattn_partial_fwd(q, k, v, q_pos, kv_pos, scale, causal, kv_valid)

    def merge(self, o_acc, lse_acc, o_blk, lse_blk):
        return self._r.rattn_merge(o_acc, lse_acc, o_blk, lse_blk)

    def prep(self, o, do):
        return self._r.rattn_bwd_prep(o, do)

    def bwd(self, q, k, v, do, lse, delta, q_pos, kv_pos, scale, causal, kv_valid, dq_acc, dk=None, dv=None):
        return self._r.rattn_partial_bwd(q, k, v, do, lse, delta, q_pos, kv_pos, dq_acc, scale, causal, kv_valid,
                                         dk, dv)

    def fold(self, acc, blk):
        return self._r.rattn_grad_fold(acc, blk)


def ring_peers(group=None):
    """(rank, cp, next, prev): this process's rank in ``group``, the group's
    size, and the global ranks of the next and previous members of the ring."""
    rank = dist.get_rank(group)
    cp = dist.get_world_size(group)
    nxt, prv = (rank + 1) % cp, (rank - 1) % cp
    if group is not None:
        nxt, prv = dist.get_global_rank(group, nxt), dist.get_global_rank(group, prv)
    return rank, cp, nxt, prv


def rank_slice(x, rank, cp):
    """Rows [rank L_loc, (rank+1) L_loc) of a permuted [B, H, Lp, D] tensor (or
    of an [Lp] position array), as a contiguous copy: what rank ``rank`` holds."""
    n = x.shape[-2] if x.dim() >= 2 else x.shape[0]
    if n % cp:
        raise ValueError(f"length {n} is not a multiple of cp = {cp}")
    L_loc = n // cp
    if x.dim() >= 2:
        return x[..., rank * L_loc:(rank + 1) * L_loc, :].contiguous()
    return x[rank * L_loc:(rank + 1) * L_loc].contiguous()


def _check_local(q, k, v, pos):
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError(f"q, k, v must share one [B, H, L_loc, D] shape, got {tuple(q.shape)}, "
                         f"{tuple(k.shape)}, {tuple(v.shape)}")
    if pos.dim() != 1 or pos.shape[0] != q.shape[2] or pos.dtype != torch.int32:
        raise ValueError(f"pos must be int32 [L_loc = {q.shape[2]}], got {pos.dtype} {tuple(pos.shape)}")
    for t in (q, k, v, pos):
        if not t.is_contiguous() or t.device != q.device:
            raise ValueError("q, k, v and pos must be contiguous and on one device")


def _exchange(sends, recvs, nxt, prv, tag, group):
    ops = [dist.P2POp(dist.isend, t, nxt, group, tag) for t in sends]
    ops += [dist.P2POp(dist.irecv, t, prv, group, tag) for t in recvs]
    return dist.batch_isend_irecv(ops)


def _wait(reqs):
    for r in reqs:
        r.wait()


def _scale(q, scale):
    return q.shape[-1] ** -0.5 if scale is None else float(scale)


def ring_fwd(q, k, v, pos, scale=None, causal=True, kv_valid=2 ** 62, group=None, ops=None):
    """This rank's rows of the ring forward over the processes of ``group``.

    q, k, v: [B, H, L_loc, D], the rank's slice of the permuted sequence; pos:
    int32 [L_loc], its global positions (non-decreasing). Keys with position
    >= kv_valid are masked (the sequence's pad rows). Returns O and LSE of the
    rank's queries over the whole sequence, in the accumulator precision of
    ``ops`` (fp32 with ``KernelOps``)."""
    _check_local(q, k, v, pos)
    ops = KernelOps() if ops is None else ops
    scale = _scale(q, scale)
    rank, cp, nxt, prv = ring_peers(group)
    bufs = [[torch.empty_like(t) for t in (k, v, pos)] for _ in range(min(2, cp - 1))]
    cur = [k, v, pos]
    o = lse = None
    for t in range(cp):
        reqs = None
        if t < cp - 1:
            recv = bufs[t % 2]
            reqs = _exchange(cur, recv, nxt, prv, _TAG_KV, group)
        ob, lb = ops.fwd(q, cur[0], cur[1], pos, cur[2], scale, causal, kv_valid)
        if o is None:
            o, lse = ob, lb
        else:
            o, lse = ops.merge(o, lse, ob, lb)
        if reqs is not None:
            _wait(reqs)
            cur = recv
    return o, lse


def ring_bwd(q, k, v, o, do, lse, pos, scale=None, causal=True, kv_valid=2 ** 62, group=None, ops=None):
    """Gradients of ``ring_fwd`` for this rank's rows: dQ of its queries and
    dK, dV of its own key/value rows, summed over every rank's queries.

    q, k, v, do: [B, H, L_loc, D]; o: the forward output of these rows in the
    inputs' dtype (as the model keeps it) and lse its fp32 LSE; pos as in
    ``ring_fwd``. The running dK, dV sums travel one hop behind the K/V
    blocks. Returns (dq, dk, dv) in the accumulator precision of ``ops``
    (fp32 with ``KernelOps``)."""
    _check_local(q, k, v, pos)
    ops = KernelOps() if ops is None else ops
    scale = _scale(q, scale)
    rank, cp, nxt, prv = ring_peers(group)
    delta, dq = ops.prep(o, do)
    kv_bufs = [[torch.empty_like(t) for t in (k, v, pos)] for _ in range(min(2, cp - 1))]
    cur = [k, v, pos]
    shares = [None, None]          # this rank's (dk, dv) totals sent at hops t and t-1
    in_bufs = [None, None]         # running sums received for the next hop
    pending = None                 # the dK/dV exchange posted at the end of the previous hop
    for t in range(cp):
        kv_reqs = None
        if t < cp - 1:
            recv = kv_bufs[t % 2]
            kv_reqs = _exchange(cur, recv, nxt, prv, _TAG_KV, group)
        # the buffers of hop t-2, whose send completed at hop t-1's wait
        reuse = shares[t % 2] if shares[t % 2] is not None else (None, None)
        gk, gv = ops.bwd(q, cur[0], cur[1], do, lse, delta, pos, cur[2], scale, causal, kv_valid, dq, *reuse)
        if pending is not None:
            _wait(pending)
            dk_in, dv_in = in_bufs[(t - 1) % 2]
            ops.fold(gk, dk_in)
            ops.fold(gv, dv_in)
        shares[t % 2] = (gk, gv)
        if cp > 1:
            if in_bufs[t % 2] is None:
                in_bufs[t % 2] = (torch.empty_like(gk), torch.empty_like(gv))
            pending = _exchange([gk, gv], list(in_bufs[t % 2]), nxt, prv, _TAG_DKV, group)
        if kv_reqs is not None:
            _wait(kv_reqs)
            cur = recv
    if cp == 1:
        return (dq,) + shares[0]
    _wait(pending)
    dk, dv = in_bufs[(cp - 1) % 2]
    return dq, dk, dv


def _gather(x, cp, group):
    out = torch.empty((cp,) + tuple(x.shape), dtype=x.dtype, device=x.device)
    flat = out.view((cp * x.shape[0],) + tuple(x.shape[1:])) if x.dim() > 0 else out
    work = dist.all_gather_into_tensor(flat, x, group=group, async_op=True)
    return out, work


def allgather_fwd(q, k, v, pos, scale=None, causal=True, kv_valid=2 ** 62, group=None, ops=None):
    """``ring_fwd`` with the all-gather exchange: K, V and positions of every
    rank are gathered once (while the local block is computed) and the blocks
    folded in ring order. Same arguments and results as ``ring_fwd``, bit for
    bit; memory per rank grows to the whole sequence's K/V."""
    _check_local(q, k, v, pos)
    ops = KernelOps() if ops is None else ops
    scale = _scale(q, scale)
    rank, cp, _, _ = ring_peers(group)
    if cp == 1:
        return ops.fwd(q, k, v, pos, pos, scale, causal, kv_valid)
    (kg, wk), (vg, wv), (pg, wp) = (_gather(t, cp, group) for t in (k, v, pos))
    o, lse = ops.fwd(q, k, v, pos, pos, scale, causal, kv_valid)
    _wait([wk, wv, wp])
    for t in range(1, cp):
        s = (rank - t) % cp
        ob, lb = ops.fwd(q, kg[s], vg[s], pos, pg[s], scale, causal, kv_valid)
        o, lse = ops.merge(o, lse, ob, lb)
    return o, lse


def allgather_bwd(q, k, v, o, do, lse, pos, scale=None, causal=True, kv_valid=2 ** 62, group=None, ops=None):
    """Gradients of ``allgather_fwd``: every rank computes its queries' share
    of dK, dV for every block, and one reduce-scatter returns to each rank the
    sum for its own block. Same arguments and results as ``ring_bwd`` (up to
    the order of the dK, dV sums)."""
    _check_local(q, k, v, pos)
    ops = KernelOps() if ops is None else ops
    scale = _scale(q, scale)
    rank, cp, _, _ = ring_peers(group)
    delta, dq = ops.prep(o, do)
    if cp == 1:
        return (dq,) + tuple(ops.bwd(q, k, v, do, lse, delta, pos, pos, scale, causal, kv_valid, dq))
    (kg, wk), (vg, wv), (pg, wp) = (_gather(t, cp, group) for t in (k, v, pos))
    dkg = torch.empty((cp,) + tuple(k.shape), dtype=dq.dtype, device=dq.device)   # every block's shares
    dvg = torch.empty_like(dkg)
    ops.bwd(q, k, v, do, lse, delta, pos, pos, scale, causal, kv_valid, dq, dkg[rank], dvg[rank])
    _wait([wk, wv, wp])
    for t in range(1, cp):
        s = (rank - t) % cp
        ops.bwd(q, kg[s], vg[s], do, lse, delta, pos, pg[s], scale, causal, kv_valid, dq, dkg[s], dvg[s])
    dk, dv = torch.empty_like(dkg[0]), torch.empty_like(dvg[0])
    for out, full in ((dk, dkg), (dv, dvg)):
        dist.reduce_scatter_tensor(out, full.view((cp * out.shape[0],) + tuple(out.shape[1:])), group=group)
    return dq, dk, dv
