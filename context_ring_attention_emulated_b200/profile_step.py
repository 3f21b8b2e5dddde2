"""Runs the hot path on a chosen size for profilers (ncu): permute, ring
forward, ring backward, merge, a few times on seeded inputs.

  python -m context_ring_attention_emulated_b200.profile_step --H 32 --L 16000 --cp 4 --iters 2

Each iteration launches, in order: 4 permutes (q, k, v, dO), ring fwd,
unpermute O, ring bwd (prep, main, dQ convert), 3 unpermutes, one merge
(fp32 O and LSE of the ring forward folded into a copy of themselves).
"""
import argparse
import sys

import torch

from . import rattn
from .workloads import make_tensor


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--B", type=int, default=1)
    ap.add_argument("--H", type=int, default=32)
    ap.add_argument("--L", type=int, default=16000)
    ap.add_argument("--D", type=int, default=128)
    ap.add_argument("--cp", type=int, default=4)
    ap.add_argument("--layout", type=int, default=rattn.LAYOUT_HEAD_TAIL)
    ap.add_argument("--noncausal", action="store_true")
    ap.add_argument("--iters", type=int, default=2)
    ap.add_argument("--fwd-tiling", type=int, default=0, help="rattn_set_fwd_tiling mode (0 automatic)")
    a = ap.parse_args(argv)
    rattn.rattn_set_fwd_tiling(a.fwd_tiling)
    causal = not a.noncausal
    shape = (a.B, a.H, a.L, a.D)
    q, k, v, do = (make_tensor(shape, torch.bfloat16, "cuda", seed=s) for s in range(4))
    o_acc = torch.zeros(a.B, a.H, a.L, a.D, dtype=torch.float32, device="cuda")
    l_acc = torch.full((a.B, a.H, a.L), float("-inf"), dtype=torch.float32, device="cuda")
    o_blk = make_tensor(shape, torch.float32, "cuda", seed=5)
    l_blk = make_tensor(shape[:3], torch.float32, "cuda", seed=6)
    for _ in range(a.iters):
        qp, pos = rattn.cp_layout_permute(q, a.cp, a.layout)
        kp, _ = rattn.cp_layout_permute(k, a.cp, a.layout)
        vp, _ = rattn.cp_layout_permute(v, a.cp, a.layout)
        dop, _ = rattn.cp_layout_permute(do, a.cp, a.layout)
        o, lse = rattn.rattn_ring_fwd(qp, kp, vp, pos, a.cp, a.layout, causal, L_valid=a.L)
        rattn.cp_layout_unpermute(o, a.L, a.cp, a.layout)
        dq, dk, dv = rattn.rattn_ring_bwd(qp, kp, vp, o, dop, lse, pos, a.cp, a.layout, causal, L_valid=a.L)
        for g in (dq, dk, dv):
            rattn.cp_layout_unpermute(g, a.L, a.cp, a.layout)
        rattn.rattn_merge(o_acc, l_acc, o_blk, l_blk)
    torch.cuda.synchronize()
    code, site = rattn.rattn_get_device_error()
    if code != rattn.OK:
        print(f"device wait timed out at site {site}", file=sys.stderr)
        return 1
    print("ok")
    return 0


if __name__ == "__main__":
    sys.exit(main())
