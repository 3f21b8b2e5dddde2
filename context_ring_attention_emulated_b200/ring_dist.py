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
kernels: ``rattn_partial_fwd_gqa`` and ``rattn_merge`` in the forward (O and LSE
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
same cp, shapes and dtypes). A group whose backend moves only host memory
(gloo) can still carry CUDA blocks: each exchange then copies the blocks it
sends into pinned host buffers, moves those, and copies what arrives back to
the device on the current stream when the exchange is waited for.

Grouped key/value heads: K and V may have H_kv heads with H a multiple of
H_kv (query head h reads key/value head h / (H / H_kv)); only the H_kv heads
travel, which is what makes the ring's traffic O(L H_kv) in [Megatron-CP].

Each hop's work is bracketed by an NVTX range ("rattn hop t") when the
tensors are on a GPU, so a profiler's timeline shows the hops.

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
        return self._r.rattn_partial_fwd_gqa(q, k, v, q_pos, kv_pos, scale, causal, kv_valid)

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
    if q.dim() != 4 or k.dim() != 4 or v.shape != k.shape:
        raise ValueError(f"q must be [B, H, L_loc, D] and k, v one [B, H_kv, L_loc, D] shape, got "
                         f"{tuple(q.shape)}, {tuple(k.shape)}, {tuple(v.shape)}")
    B, H, L_loc, D = q.shape
    H_kv = k.shape[1]
    if k.shape[0] != B or k.shape[2] != L_loc or k.shape[3] != D or H_kv < 1 or H % H_kv:
        raise ValueError(f"k, v must be [B={B}, H_kv, L_loc={L_loc}, D={D}] with H={H} a multiple of H_kv, "
                         f"got {tuple(k.shape)}")
    if pos.dim() != 1 or pos.shape[0] != L_loc or pos.dtype != torch.int32:
        raise ValueError(f"pos must be int32 [L_loc = {L_loc}], got {pos.dtype} {tuple(pos.shape)}")
    for t in (q, k, v, pos):
        if not t.is_contiguous() or t.device != q.device:
            raise ValueError("q, k, v and pos must be contiguous and on one device")


def _host_staged(group, tensors):
    """True when the group's backend moves host memory only (gloo) and some of
    the tensors live on a GPU: they then travel through pinned host copies."""
    return dist.get_backend(group) == "gloo" and any(t.is_cuda for t in tensors)


def _to_host(t):
    """Pinned host copy of a device tensor, complete when this returns."""
    h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
    h.copy_(t)
    return h


def _wire(t):
    """The bytes of a contiguous tensor, as the exchange moves them."""
    return t.reshape(-1).view(torch.uint8)


class _Exchange:
    """One posted exchange: ``sends`` go to rank ``nxt`` and ``recvs`` are
    filled from rank ``prv``; ``wait()`` completes it."""

    def __init__(self, sends, recvs, nxt, prv, tag, group):
        self.recvs = recvs
        self.host_recvs = None
        if _host_staged(group, list(sends) + list(recvs)):
            sends = [_to_host(t) for t in sends]
            self.host_recvs = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in recvs]
            recvs = self.host_recvs
        self._keep = sends
        ops = [dist.P2POp(dist.isend, _wire(t), nxt, group, tag) for t in sends]
        ops += [dist.P2POp(dist.irecv, _wire(t), prv, group, tag) for t in recvs]
        self.reqs = dist.batch_isend_irecv(ops)

    def wait(self):
        for r in self.reqs:
            r.wait()
        if self.host_recvs is not None:
            for d, h in zip(self.recvs, self.host_recvs):
                d.copy_(h, non_blocking=True)
            self.host_recvs = None


def _exchange(sends, recvs, nxt, prv, tag, group):
    return _Exchange(sends, recvs, nxt, prv, tag, group)


def _wait(reqs):
    for r in reqs:
        r.wait()


class _hop:
    """NVTX range around one hop's work when the tensors are on a GPU."""

    def __init__(self, t, on_gpu):
        self.t, self.on_gpu = t, on_gpu

    def __enter__(self):
        if self.on_gpu:
            torch.cuda.nvtx.range_push(f"rattn hop {self.t}")

    def __exit__(self, *a):
        if self.on_gpu:
            torch.cuda.nvtx.range_pop()


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
        with _hop(t, q.is_cuda):
            xch = None
            if t < cp - 1:
                recv = bufs[t % 2]
                xch = _exchange(cur, recv, nxt, prv, _TAG_KV, group)
            ob, lb = ops.fwd(q, cur[0], cur[1], pos, cur[2], scale, causal, kv_valid)
            if o is None:
                o, lse = ob, lb
            else:
                o, lse = ops.merge(o, lse, ob, lb)
            if xch is not None:
                xch.wait()
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
        with _hop(t, q.is_cuda):
            kv_xch = None
            if t < cp - 1:
                recv = kv_bufs[t % 2]
                kv_xch = _exchange(cur, recv, nxt, prv, _TAG_KV, group)
            # the buffers of hop t-2, whose send completed at hop t-1's wait
            reuse = shares[t % 2] if shares[t % 2] is not None else (None, None)
            gk, gv = ops.bwd(q, cur[0], cur[1], do, lse, delta, pos, cur[2], scale, causal, kv_valid, dq, *reuse)
            if pending is not None:
                pending.wait()
                dk_in, dv_in = in_bufs[(t - 1) % 2]
                ops.fold(gk, dk_in)
                ops.fold(gv, dv_in)
            shares[t % 2] = (gk, gv)
            if cp > 1:
                if in_bufs[t % 2] is None:
                    in_bufs[t % 2] = (torch.empty_like(gk), torch.empty_like(gv))
                pending = _exchange([gk, gv], list(in_bufs[t % 2]), nxt, prv, _TAG_DKV, group)
            if kv_xch is not None:
                kv_xch.wait()
                cur = recv
    if cp == 1:
        return (dq,) + shares[0]
    pending.wait()
    dk, dv = in_bufs[(cp - 1) % 2]
    return dq, dk, dv


class _Gather:
    """All ranks' copies of ``x`` stacked as [cp, *x.shape], gathered
    asynchronously; ``wait()`` completes it (host-staged on gloo)."""

    def __init__(self, x, cp, group):
        self.out = torch.empty((cp,) + tuple(x.shape), dtype=x.dtype, device=x.device)
        self.host = None
        src, dst = x, self.out
        if _host_staged(group, [x]):
            src = _to_host(x)
            self.host = dst = torch.empty(self.out.shape, dtype=x.dtype, pin_memory=True)
        self.work = dist.all_gather_into_tensor(_wire(dst), _wire(src), group=group, async_op=True)
        self._keep = src

    def wait(self):
        self.work.wait()
        if self.host is not None:
            self.out.copy_(self.host, non_blocking=True)
            self.host = None


def _reduce_scatter(out, full, group):
    """out = this rank's block of the sum over ranks of ``full`` [cp * n, ...]."""
    if _host_staged(group, [out, full]):
        h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        dist.reduce_scatter_tensor(h, _to_host(full), group=group)
        out.copy_(h, non_blocking=True)
    else:
        dist.reduce_scatter_tensor(out, full, group=group)


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
    gathers = [_Gather(t, cp, group) for t in (k, v, pos)]
    with _hop(0, q.is_cuda):
        o, lse = ops.fwd(q, k, v, pos, pos, scale, causal, kv_valid)
    _wait(gathers)
    kg, vg, pg = (g.out for g in gathers)
    for t in range(1, cp):
        s = (rank - t) % cp
        with _hop(t, q.is_cuda):
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
    gathers = [_Gather(t, cp, group) for t in (k, v, pos)]
    dkg = torch.empty((cp,) + tuple(k.shape), dtype=dq.dtype, device=dq.device)   # every block's shares
    dvg = torch.empty_like(dkg)
    with _hop(0, q.is_cuda):
        ops.bwd(q, k, v, do, lse, delta, pos, pos, scale, causal, kv_valid, dq, dkg[rank], dvg[rank])
    _wait(gathers)
    kg, vg, pg = (g.out for g in gathers)
    for t in range(1, cp):
        s = (rank - t) % cp
        with _hop(t, q.is_cuda):
            ops.bwd(q, kg[s], vg[s], do, lse, delta, pos, pg[s], scale, causal, kv_valid, dq, dkg[s], dvg[s])
    dk, dv = torch.empty_like(dkg[0]), torch.empty_like(dvg[0])
    for out, full in ((dk, dkg), (dv, dvg)):
        _reduce_scatter(out, full.view((cp * out.shape[0],) + tuple(out.shape[1:])), group)
    return dq, dk, dv
