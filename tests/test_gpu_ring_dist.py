"""The ring across processes, one CP rank per process, with this library's
CUDA kernels as the block arithmetic and a real exchange between the ranks.

Pages: the Ultralytics glossary "Context Parallelism", section "How context
parallelism works" (each device computes a partial attention on the K/V block
it holds, passes the block to the next device and repeats), and the blog
"Context Parallelism v.s. Sequence Parallelism (Megatron-LM)", section "CP vs
SP" (K/V move ring-style by point-to-point sends or by an all-gather; the
traffic is sized by the key/value heads).

cp = 2 and cp = 4 processes share the one GPU of this machine and exchange
over a gloo group: every K/V block, position array and running dK/dV sum
crosses between processes (through pinned host copies, as ``ring_dist`` does
for a gloo group). No kernel waits on another process: each rank's kernels
run on its own data, and the exchange happens on the host between them.
Every rank runs ``ring_fwd``, ``allgather_fwd``, ``ring_bwd`` and
``allgather_bwd``; the rows of all ranks, put back in global order, are
compared with the oracle's attention and gradient of the whole sequence at
the bf16 tolerances. Cases cover a padded length, the striped layout, the
contiguous non-causal layout, grouped key/value heads and D = 64."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from tests.gpu_common import check_grad, check_lse, check_o

pytestmark = pytest.mark.gpu

HEAD_TAIL, STRIPED, CONTIGUOUS = 1, 2, 0
# (cp, L, H, H_kv, D, layout, causal)
CASES = [
    (2, 1024, 2, 2, 128, HEAD_TAIL, True),
    (4, 998, 4, 2, 128, HEAD_TAIL, True),     # padded to 1000; grouped key/value heads
    (4, 1024, 2, 2, 64, STRIPED, True),
    (2, 700, 2, 1, 128, CONTIGUOUS, False),   # one key/value head for both query heads
]


def _inputs(L, H, H_kv, D, seed):
    from context_ring_attention_emulated_b200.workloads import make_tensor
    shapes = ((1, H, L, D), (1, H_kv, L, D), (1, H_kv, L, D), (1, H, L, D))
    return [make_tensor(s, torch.bfloat16, "cpu", seed=seed + i) for i, s in enumerate(shapes)]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, cases, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        from context_ring_attention_emulated_b200 import rattn, ring_dist
        for i, (cp, L, H, H_kv, D, layout, causal) in enumerate(cases):
            q, k, v, do = (x.cuda() for x in _inputs(L, H, H_kv, D, 100 * i))
            qp, pos = rattn.cp_layout_permute(q, cp, layout)
            kp, _ = rattn.cp_layout_permute(k, cp, layout)
            vp, _ = rattn.cp_layout_permute(v, cp, layout)
            dop, _ = rattn.cp_layout_permute(do, cp, layout)
            ql, kl, vl, dol = (ring_dist.rank_slice(x, rank, cp) for x in (qp, kp, vp, dop))
            pl = ring_dist.rank_slice(pos, rank, cp)
            scale = D ** -0.5
            o, lse = ring_dist.ring_fwd(ql, kl, vl, pl, scale, causal, L)
            o2, lse2 = ring_dist.allgather_fwd(ql, kl, vl, pl, scale, causal, L)
            ob = o.to(torch.bfloat16)
            dq, dk, dv = ring_dist.ring_bwd(ql, kl, vl, ob, dol, lse, pl, scale, causal, L)
            g2 = ring_dist.allgather_bwd(ql, kl, vl, ob, dol, lse, pl, scale, causal, L)
            torch.cuda.synchronize()
            err = rattn.rattn_get_device_error()[0]
            torch.save({"o": o.cpu(), "lse": lse.cpu(), "same": bool(torch.equal(o, o2) and torch.equal(lse, lse2)),
                        "dq": dq.cpu(), "dk": dk.cpu(), "dv": dv.cpu(), "ag": [x.cpu() for x in g2], "err": err},
                       os.path.join(outdir, f"r{rank}_c{i}.pt"))
    finally:
        dist.destroy_process_group()


def _assemble(parts, L, cp, layout):
    """The ranks' rows in rank-major order, put back in global order."""
    full = torch.cat(parts, dim=-2 if parts[0].dim() == 4 else -1).double().numpy()
    if full.ndim == 3:
        return oracle.unpermute(full[..., None], L, cp, layout)[..., 0]
    return oracle.unpermute(full, L, cp, layout)


@pytest.mark.parametrize("world", [2, 4])
def test_ring_across_processes_matches_full_attention(world, tmp_path):
    cases = [c for c in CASES if c[0] == world]
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, cases, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=600)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    for i, (cp, L, H, H_kv, D, layout, causal) in enumerate(cases):
        res = [torch.load(os.path.join(tmp_path, f"r{r}_c{i}.pt")) for r in range(cp)]
        assert all(x["err"] == 0 for x in res), "a device-side wait gave up"
        assert all(x["same"] for x in res), "all-gather forward differs from the ring's"
        q, k, v, do = (x.double().numpy() for x in _inputs(L, H, H_kv, D, 100 * i))
        ke, ve = oracle.gqa_expand(k, H), oracle.gqa_expand(v, H)
        scale = D ** -0.5
        o_ref, lse_ref = oracle.attention(q, ke, ve, scale, causal)
        dq_ref, dke, dve = oracle.attention_bwd(q, ke, ve, do, scale, causal)
        refs = {"dq": dq_ref, "dk": oracle.gqa_reduce(dke, H_kv), "dv": oracle.gqa_reduce(dve, H_kv)}
        get = lambda name: _assemble([x[name] for x in res], L, cp, layout)
        check_o(get("o"), o_ref, torch.bfloat16)
        check_lse(get("lse"), lse_ref, torch.bfloat16)
        for name in ("dq", "dk", "dv"):
            check_grad(get(name), refs[name])
        for j, name in enumerate(("dq", "dk", "dv")):
            check_grad(_assemble([x["ag"][j] for x in res], L, cp, layout), refs[name])
