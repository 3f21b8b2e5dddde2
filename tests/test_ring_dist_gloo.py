"""The multi-process ring (one CP rank per process) on CPU gloo ranks.

The exchange schedules of ``ring_dist`` run over 2, 3 and 4 processes with the
fp64 oracle as their block arithmetic (the library's kernels need a GPU; the
schedule is what is under test here). Each rank holds its slice of the
permuted sequence; the rows of all ranks, put back in global order, must equal
the oracle's attention and gradient of the whole sequence, for every layout,
with and without the causal mask and with pad rows. The all-gather variant
must give the ring's forward bit for bit. Ranks that leave are seen on the
host, before or during the next exchange, never by a hang."""
import datetime
import os
import socket
import time

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from context_ring_attention_emulated_b200 import ring_dist


class OracleOps:
    """The block arithmetic of the schedules, from the fp64 oracle (tests
    only), with the interface of ``ring_dist.KernelOps``."""

    def fwd(self, q, k, v, q_pos, kv_pos, scale, causal, kv_valid):
        H = q.shape[1]
        k, v = (oracle.gqa_expand(x.numpy(), H) for x in (k, v))
        o, lse = oracle.attention(q.numpy(), k, v, scale, causal, q_pos.numpy(), kv_pos.numpy(), kv_valid)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def merge(self, o_acc, lse_acc, o_blk, lse_blk):
        o, lse = oracle.merge(o_acc.numpy(), lse_acc.numpy(), o_blk.numpy(), lse_blk.numpy())
        return torch.from_numpy(o), torch.from_numpy(lse)

    def prep(self, o, do):
        delta = torch.from_numpy((o.numpy().astype(np.float64) * do.numpy()).sum(-1))
        return delta, torch.zeros(do.shape, dtype=torch.float64)

    def bwd(self, q, k, v, do, lse, delta, q_pos, kv_pos, scale, causal, kv_valid, dq_acc, dk=None, dv=None):
        H, H_kv = q.shape[1], k.shape[1]
        ke, ve = (oracle.gqa_expand(x.numpy(), H) for x in (k, v))
        gq, gk, gv = oracle.attention_bwd_block(q.numpy(), ke, ve, do.numpy(), lse.numpy(), delta.numpy(), scale,
                                                causal, q_pos.numpy(), kv_pos.numpy(), kv_valid)
        gk, gv = oracle.gqa_reduce(gk, H_kv), oracle.gqa_reduce(gv, H_kv)
        gq, gk, gv = (torch.from_numpy(np.ascontiguousarray(x)) for x in (gq, gk, gv))
        dq_acc += gq
        if dk is None:
            return gk, gv
        dk.copy_(gk)
        dv.copy_(gv)
        return dk, dv

    def fold(self, acc, blk):
        acc += blk
        return acc


LAYOUTS = (oracle.CONTIGUOUS, oracle.HEAD_TAIL, oracle.STRIPED)
B, H, D, SCALE = 1, 2, 4, 0.55


def _configs(cp):
    """(layout, causal, L): every layout, both masks, an exact and a padded length."""
    out = []
    for layout in LAYOUTS:
        for causal in (True, False):
            for L in (6 * cp, 6 * cp - 3):
                out.append((layout, causal, L))
    return out


def _inputs(L, seed):
    g = np.random.default_rng(seed)
    return [g.standard_normal((B, H, L, D)) for _ in range(4)]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port, timeout_s=60):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=timeout_s))


def _rank_main(rank, world, port, out):
    _init(rank, world, port)
    ops = OracleOps()
    try:
        for i, (layout, causal, L) in enumerate(_configs(world)):
            q, k, v, do = _inputs(L, 100 * world + i)
            Lp, _, pos = oracle.perm_index(L, world, layout)
            qp, kp, vp, dop = (torch.from_numpy(oracle.permute(x, world, layout)[0]) for x in (q, k, v, do))
            pos_t = torch.from_numpy(np.asarray(pos, dtype=np.int32))
            ql, kl, vl, dol = (ring_dist.rank_slice(x, rank, world) for x in (qp, kp, vp, dop))
            pl = ring_dist.rank_slice(pos_t, rank, world)
            o, lse = ring_dist.ring_fwd(ql, kl, vl, pl, SCALE, causal, L, ops=ops)
            o2, lse2 = ring_dist.allgather_fwd(ql, kl, vl, pl, SCALE, causal, L, ops=ops)
            dq, dk, dv = ring_dist.ring_bwd(ql, kl, vl, o, dol, lse, pl, SCALE, causal, L, ops=ops)
            g2 = ring_dist.allgather_bwd(ql, kl, vl, o, dol, lse, pl, SCALE, causal, L, ops=ops)
            same = bool(torch.equal(o, o2) and torch.equal(lse, lse2))
            out[(rank, i)] = dict(o=o.numpy(), lse=lse.numpy(), same=same, dq=dq.numpy(), dk=dk.numpy(),
                                  dv=dv.numpy(), ag=[x.numpy() for x in g2])
    finally:
        dist.destroy_process_group()


def _assemble(parts, L, cp, layout):
    """Concatenate the ranks' rows (rank-major order) and return them in global order."""
    full = np.concatenate(parts, axis=-2 if parts[0].ndim == 4 else -1)
    if full.ndim == 3:
        return oracle.unpermute(full[..., None], L, cp, layout)[..., 0]
    return oracle.unpermute(full, L, cp, layout)


@pytest.mark.parametrize("world", [2, 3, 4])
def test_ring_and_allgather_match_full_attention(world):
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for i, (layout, causal, L) in enumerate(_configs(world)):
        q, k, v, do = _inputs(L, 100 * world + i)
        o_ref, lse_ref = oracle.attention(q, k, v, SCALE, causal)
        dq_ref, dk_ref, dv_ref = oracle.attention_bwd(q, k, v, do, SCALE, causal)
        ranks = [res[(r, i)] for r in range(world)]
        assert all(x["same"] for x in ranks), "all-gather forward differs from the ring's"
        get = lambda name: _assemble([x[name] for x in ranks], L, world, layout)
        np.testing.assert_allclose(get("o"), o_ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(get("lse"), lse_ref, rtol=0, atol=1e-12)
        for name, ref in (("dq", dq_ref), ("dk", dk_ref), ("dv", dv_ref)):
            np.testing.assert_allclose(get(name), ref, rtol=0, atol=1e-12, err_msg=f"{name} {layout} {causal} {L}")
        for j, ref in enumerate((dq_ref, dk_ref, dv_ref)):
            ag = _assemble([x["ag"][j] for x in ranks], L, world, layout)
            np.testing.assert_allclose(ag, ref, rtol=0, atol=1e-12)


GQA_HEADS = ((4, 2), (4, 1))   # (H, H_kv)


def _gqa_inputs(L, H, H_kv, seed):
    g = np.random.default_rng(seed)
    shapes = ((B, H, L, D), (B, H_kv, L, D), (B, H_kv, L, D), (B, H, L, D))
    return [g.standard_normal(s) for s in shapes]


def _gqa_main(rank, world, port, out):
    """The ring and all-gather schedules with K, V on fewer heads than Q: only
    the H_kv heads travel, and dK, dV come back summed over each group."""
    _init(rank, world, port)
    ops = OracleOps()
    try:
        for i, (H, H_kv) in enumerate(GQA_HEADS):
            L = 6 * world - 1
            q, k, v, do = _gqa_inputs(L, H, H_kv, 300 + 10 * world + i)
            _, _, pos = oracle.perm_index(L, world, oracle.HEAD_TAIL)
            qp, kp, vp, dop = (torch.from_numpy(oracle.permute(x, world, oracle.HEAD_TAIL)[0]) for x in (q, k, v, do))
            pl = ring_dist.rank_slice(torch.from_numpy(np.asarray(pos, dtype=np.int32)), rank, world)
            ql, kl, vl, dol = (ring_dist.rank_slice(x, rank, world) for x in (qp, kp, vp, dop))
            o, lse = ring_dist.ring_fwd(ql, kl, vl, pl, SCALE, True, L, ops=ops)
            dq, dk, dv = ring_dist.ring_bwd(ql, kl, vl, o, dol, lse, pl, SCALE, True, L, ops=ops)
            g2 = ring_dist.allgather_bwd(ql, kl, vl, o, dol, lse, pl, SCALE, True, L, ops=ops)
            out[(rank, i)] = dict(o=o.numpy(), dq=dq.numpy(), dk=dk.numpy(), dv=dv.numpy(),
                                  ag=[x.numpy() for x in g2])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ring_carries_grouped_kv_heads(world):
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_gqa_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for i, (H, H_kv) in enumerate(GQA_HEADS):
        L = 6 * world - 1
        q, k, v, do = _gqa_inputs(L, H, H_kv, 300 + 10 * world + i)
        ke, ve = oracle.gqa_expand(k, H), oracle.gqa_expand(v, H)
        o_ref, _ = oracle.attention(q, ke, ve, SCALE, True)
        dq_ref, dke, dve = oracle.attention_bwd(q, ke, ve, do, SCALE, True)
        refs = {"dq": dq_ref, "dk": oracle.gqa_reduce(dke, H_kv), "dv": oracle.gqa_reduce(dve, H_kv)}
        ranks = [res[(r, i)] for r in range(world)]
        get = lambda name: _assemble([x[name] for x in ranks], L, world, oracle.HEAD_TAIL)
        np.testing.assert_allclose(get("o"), o_ref, rtol=0, atol=1e-12)
        for name, ref in refs.items():
            np.testing.assert_allclose(get(name), ref, rtol=0, atol=1e-12, err_msg=f"{name} H={H} H_kv={H_kv}")
        for j, name in enumerate(("dq", "dk", "dv")):
            ag = _assemble([x["ag"][j] for x in ranks], L, world, oracle.HEAD_TAIL)
            np.testing.assert_allclose(ag, refs[name], rtol=0, atol=1e-12)


def _subgroup_main(rank, world, port, out):
    """Two rings at once on four processes: {0, 2} and {1, 3} (CP groups
    inside a larger job); each must exchange only within its own group."""
    _init(rank, world, port)
    try:
        groups = [dist.new_group([0, 2]), dist.new_group([1, 3])]
        g = groups[rank % 2]
        cp, gr = 2, dist.get_rank(g)
        L = 10
        q, k, v, do = _inputs(L, 700 + rank % 2)           # each ring its own sequence
        Lp, _, pos = oracle.perm_index(L, cp, oracle.HEAD_TAIL)
        qp, kp, vp, dop = (torch.from_numpy(oracle.permute(x, cp, oracle.HEAD_TAIL)[0]) for x in (q, k, v, do))
        pl = ring_dist.rank_slice(torch.from_numpy(np.asarray(pos, dtype=np.int32)), gr, cp)
        ql, kl, vl, dol = (ring_dist.rank_slice(x, gr, cp) for x in (qp, kp, vp, dop))
        o, lse = ring_dist.ring_fwd(ql, kl, vl, pl, SCALE, True, L, group=g, ops=OracleOps())
        dq, dk, dv = ring_dist.ring_bwd(ql, kl, vl, o, dol, lse, pl, SCALE, True, L, group=g, ops=OracleOps())
        out[rank] = dict(gr=gr, o=o.numpy(), dq=dq.numpy(), dk=dk.numpy(), dv=dv.numpy())
    finally:
        dist.destroy_process_group()


def test_rings_on_subgroups_exchange_within_their_group():
    world, port = 4, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_subgroup_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for ring, members in ((0, (0, 2)), (1, (1, 3))):
        q, k, v, do = _inputs(10, 700 + ring)
        parts = sorted((res[r]["gr"], res[r]) for r in members)
        o = _assemble([p["o"] for _, p in parts], 10, 2, oracle.HEAD_TAIL)
        np.testing.assert_allclose(o, oracle.attention(q, k, v, SCALE, True)[0], rtol=0, atol=1e-12)
        for name, ref in zip(("dq", "dk", "dv"), oracle.attention_bwd(q, k, v, do, SCALE, True)):
            got = _assemble([p[name] for _, p in parts], 10, 2, oracle.HEAD_TAIL)
            np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_single_rank_ring_is_the_local_attention():
    port = _free_port()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        q, k, v, do = (torch.from_numpy(x) for x in _inputs(9, 3))
        pos = torch.arange(9, dtype=torch.int32)
        o, lse = ring_dist.ring_fwd(q, k, v, pos, SCALE, True, ops=OracleOps())
        o_ref, lse_ref = oracle.attention(q.numpy(), k.numpy(), v.numpy(), SCALE, True)
        np.testing.assert_allclose(o.numpy(), o_ref, rtol=0, atol=1e-12)
        dq, dk, dv = ring_dist.ring_bwd(q, k, v, o, do, lse, pos, SCALE, True, ops=OracleOps())
        for got, ref in zip((dq, dk, dv), oracle.attention_bwd(q.numpy(), k.numpy(), v.numpy(), do.numpy(), SCALE,
                                                                True)):
            np.testing.assert_allclose(got.numpy(), ref, rtol=0, atol=1e-12)
    finally:
        dist.destroy_process_group()


def test_kernel_ops_take_no_cpu_path():
    """The default block arithmetic is the library's CUDA kernels alone: CPU
    tensors are refused by every schedule, forward and backward."""
    port = _free_port()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        q, k, v, do = (torch.from_numpy(x).float() for x in _inputs(8, 5))
        pos = torch.arange(8, dtype=torch.int32)
        with pytest.raises(ValueError, match="CUDA"):
            ring_dist.ring_fwd(q, k, v, pos)
        with pytest.raises(ValueError, match="CUDA"):
            ring_dist.allgather_fwd(q, k, v, pos)
        with pytest.raises(ValueError, match="CUDA"):
            ring_dist.ring_bwd(q, k, v, q, do, q[..., 0], pos)
        with pytest.raises(ValueError, match="CUDA"):
            ring_dist.allgather_bwd(q, k, v, q, do, q[..., 0], pos)
        with pytest.raises(ValueError, match="int32"):
            ring_dist.ring_fwd(q, k, v, pos.long(), ops=OracleOps())
        with pytest.raises(ValueError, match="shape"):
            ring_dist.ring_fwd(q, k[:, :1], v, pos, ops=OracleOps())
    finally:
        dist.destroy_process_group()


# ---- failures are seen on the host ------------------------------------------

def _store_barrier(store, name, world):
    if store.add(name, 1) == world:
        store.set(name + "/go", "1")
    store.wait([name + "/go"])


def _member_main(rank, world, store_port, out):
    store = dist.TCPStore("127.0.0.1", store_port, world, is_master=(rank == 0),
                          timeout=datetime.timedelta(seconds=30))
    m = ring_dist.RingMembership(store, rank, world)
    m.check()                                  # everyone present: no error
    _store_barrier(store, "b0", world)
    if rank == world - 1:
        m.leave()                              # leaves between steps
    _store_barrier(store, "b1", world)
    if rank == world - 1:
        out[rank] = "left"
    else:
        try:
            m.check()
            out[rank] = "not seen"
        except ring_dist.PeerLeftError as e:
            out[rank] = e.ranks
    _store_barrier(store, "b2", world)
    if rank == 0:                              # the store's host goes last
        while store.add("bye", 0) < world - 1:
            time.sleep(0.01)
    else:
        store.add("bye", 1)


def test_membership_reports_a_rank_that_left():
    world, port = 3, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_member_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[2] == "left"
    assert res[0] == [2] and res[1] == [2]


def _dead_peer_main(rank, world, port, out):
    _init(rank, world, port, timeout_s=10)
    if rank == 1:
        out[rank] = "exited"
        os._exit(0)                            # leaves without a word, between steps
    q, k, v, _ = (torch.from_numpy(x) for x in _inputs(8, 4))
    pos = torch.arange(8 * rank, 8 * rank + 8, dtype=torch.int32)
    try:
        ring_dist.ring_fwd(q, k, v, pos, SCALE, True, ops=OracleOps())
        out[rank] = "no error"
    except RuntimeError as e:
        out[rank] = "error: " + str(e).splitlines()[0][:200]
    os._exit(0)


@pytest.mark.timeout(180)
def test_exchange_with_a_dead_peer_raises_instead_of_hanging():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_dead_peer_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        alive = [p for p in procs if p.is_alive()]
        for p in alive:
            p.kill()
        res = dict(out)
    assert not alive, "a rank hung on the exchange"
    assert res[1] == "exited"
    assert res[0].startswith("error"), res[0]


def test_test_ops_mirror_the_kernel_ops_interface():
    """The schedules tested here with OracleOps run on the GPU with KernelOps:
    both must offer the same methods with the same parameters."""
    import inspect
    names = [n for n in vars(ring_dist.KernelOps) if not n.startswith("_")]
    assert sorted(names) == ["bwd", "fold", "fwd", "merge", "prep"]
    for n in names:
        a = inspect.signature(getattr(ring_dist.KernelOps, n))
        b = inspect.signature(getattr(OracleOps, n))
        assert list(a.parameters) == list(b.parameters), n
