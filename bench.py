"""Benchmark: ring attention with emulated CP ranks on B200.

One step = the whole hot path on one batch of seeded synthetic input:
permute Q, K, V and dO to the head-tail layout, ring forward, unpermute O,
ring backward (dQ, dK, dV from the saved LSE), unpermute the gradients.
Default workload: the 32,000-token / cp=4 fwd+bwd configuration (B=1, H=32,
D=128, bf16, causal). Metric: causal-adjusted TFLOP/s of fwd + bwd
(fwd = 2*B*H*D*L^2, bwd = 2.5 x fwd).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Under torchrun (N > 1) every rank runs an independent replica of the
workload (each emulates all CP ranks on its own GPU, so no data crosses
GPUs); value is the work of all ranks over the max-over-ranks device time.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from context_ring_attention_emulated_b200.workloads import WORKLOADS, make_qkv, make_unit_grad  # noqa: E402

METRIC = "ring-attn fwd/bwd TFLOP/s (causal FLOPs) on 1 B200; % of BF16 tensor peak"
DEFAULT = "bf16_L32000_cp4_fwdbwd"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ROPE_BASE = 10000.0  # rotary base of the RoPE workloads (RoFormer's value)
# DRAM bytes (read + write) per launch of the dominant kernel, from one ncu
# capture of the current kernel on a half-length case, scaled to the full
# launch by sequence length (traffic grows with the tensors). Source:
# profiles/bwd_kernel_bf16_H32_L16000_cp4.md. Empty while the kernel has
# changed since its last capture: that capture (2.55 GB per 32k launch)
# predates the per-hop instantiation, which changed the ring instantiation's
# register allocation, so the traffic is reported as null until it is
# captured again.
NCU_TRAFFIC = {}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d, "measured"
    except OSError:
        return FALLBACK_PEAKS, "fallback"


def step_flops(w):
    fwd = w.causal_flops_fwd()
    return fwd * (3.5 if w.bwd else 1.0), fwd


def physical_gpu(local):
    """nvidia-smi index of this process's CUDA device ``local``: the entry of
    CUDA_VISIBLE_DEVICES it maps to, when that variable lists plain indices."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [v.strip() for v in vis.split(",") if v.strip()]
    if ids and local < len(ids) and ids[local].isdigit():
        return int(ids[local])
    return local


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = physical_gpu(index)
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n):
    if n <= 1 and "RANK" not in os.environ:
        return 0, 1, 0
    import datetime
    import torch.distributed as dist
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", n))
    local = int(os.environ.get("LOCAL_RANK", rank))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[torch.cuda.current_device()])
        else:
            dist.barrier()


def max_over_ranks(x, world, device="cuda"):
    """Max of a per-rank time over all ranks (every rank gets the result)."""
    if world <= 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(flops_per_step, steps, world, ms_max):
    """Whole-job throughput: the work of all ranks (each runs one replica of
    the workload) over the max-over-ranks device time."""
    return world * flops_per_step * steps / (ms_max / 1e3) / 1e12


def run_ours(args, w, rank, world, local):
    from context_ring_attention_emulated_b200 import rattn
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    q, k, v = make_qkv(w, dev, seed=0)
    do = make_unit_grad(w, dev, seed=1)
    L, cp, layout = w.L, w.cp, w.layout
    B, H, D, Hkv = w.B, w.H, w.D, w.kv_heads
    heads = {"q": H, "k": Hkv, "v": Hkv, "do": H, "o": H, "dq": H, "dk": Hkv, "dv": Hkv}
    if w.docs:  # packed sequences: host-side layout plan, index arrays resident on the device
        plan = rattn.cp_layout_varlen_plan(w.cu_seqlens, cp, layout)
        Lp = plan["Tp"]
        src, gkey, segid = (plan[n].to(dev) for n in ("src", "gkey", "segid"))
    else:
        Lp = rattn.cp_layout_padded_len(L, cp, layout)
    pbuf = {n: torch.empty(B, heads[n], Lp, D, dtype=q.dtype, device=dev) for n in ("q", "k", "v", "do", "o")}
    pos = torch.empty(Lp, dtype=torch.int32, device=dev)
    lse = torch.empty(B, H, Lp, dtype=torch.float32, device=dev)
    grads_p = [torch.empty(B, heads[n], Lp, D, dtype=q.dtype, device=dev) for n in ("dq", "dk", "dv")]
    out = {n: torch.empty(B, heads[n], L, D, dtype=q.dtype, device=dev) for n in ("o", "dq", "dk", "dv")}
    ring_fwd = rattn.rattn_ring_fwd_gqa if Hkv != H else rattn.rattn_ring_fwd
    ring_bwd = rattn.rattn_ring_bwd_gqa if Hkv != H else rattn.rattn_ring_bwd
    if w.docs:
        def ring_fwd(q_, k_, v_, pos_, cp_, layout_, causal_, scale_, L_valid=None, o=None, lse=None):
            return rattn.rattn_ring_fwd_varlen(q_, k_, v_, gkey, segid, cp_, causal_, scale_, o=o, lse=lse)

        def ring_bwd(q_, k_, v_, o_, do_, lse_, pos_, cp_, layout_, causal_, scale_, L_valid=None, dq=None, dk=None,
                     dv=None, workspace=None):
            return rattn.rattn_ring_bwd_varlen(q_, k_, v_, o_, do_, lse_, gkey, segid, cp_, causal_, scale_, dq=dq,
                                               dk=dk, dv=dv, workspace=workspace)

    def permute_in(x, name):
        if w.docs:
            rattn.cp_layout_gather(x, src, y=pbuf[name])
        elif w.rope and name in ("q", "k"):
            rattn.cp_layout_permute_rope(x, cp, layout, ROPE_BASE, rattn.ROPE_HALF, y=pbuf[name], pos=pos)
        else:
            rattn.cp_layout_permute(x, cp, layout, y=pbuf[name], pos=pos)

    def unpermute_grad(g, name, outs):  # unpermute of O and of the gradients
        if w.docs:
            rattn.cp_layout_scatter(g, src, L, x=outs[name])
        elif w.rope and name in ("dq", "dk"):
            rattn.cp_layout_unpermute_rope_grad(g, L, cp, layout, ROPE_BASE, rattn.ROPE_HALF, dx=outs[name])
        else:
            rattn.cp_layout_unpermute(g, L, cp, layout, x=outs[name])
    ws = torch.empty(max(rattn.rattn_ring_bwd_workspace_size(B, H, Lp, D), 1), dtype=torch.uint8, device=dev)
    fwd_ev, bwd_ev = [], []

    def step(x, outs=None, timed=False):
        outs = out if outs is None else outs
        xq, xk, xv, xdo = x
        permute_in(xq, "q")
        permute_in(xk, "k")
        permute_in(xv, "v")
        if timed:
            e0 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        ring_fwd(pbuf["q"], pbuf["k"], pbuf["v"], pos, cp, layout, w.causal, w.scale, L_valid=L,
                 o=pbuf["o"], lse=lse)
        if timed:
            e1 = torch.cuda.Event(enable_timing=True)
            e1.record(stream)
            fwd_ev.append((e0, e1))
        unpermute_grad(pbuf["o"], "o", outs)
        if w.bwd:
            permute_in(xdo, "do")
            if timed:
                e2 = torch.cuda.Event(enable_timing=True)
                e2.record(stream)
            ring_bwd(pbuf["q"], pbuf["k"], pbuf["v"], pbuf["o"], pbuf["do"], lse, pos, cp, layout,
                     w.causal, w.scale, L_valid=L, dq=grads_p[0], dk=grads_p[1], dv=grads_p[2],
                     workspace=ws)
            if timed:
                e3 = torch.cuda.Event(enable_timing=True)
                e3.record(stream)
                bwd_ev.append((e2, e3))
            for g, name in zip(grads_p, ("dq", "dk", "dv")):
                unpermute_grad(g, name, outs)

    launches_per_step = 3 + 1 + 1 + ((1 + 3 + 3) if w.bwd else 0)
    x = (q, k, v, do)
    for _ in range(args.warmup):
        step(x)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            step(x, timed=True)
        t1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), world)
    err, site = rattn.rattn_get_device_error()
    if err != rattn.OK:
        raise RuntimeError(f"device-side wait timed out at site {site}")
    fwd_ms = statistics.mean(a.elapsed_time(b) for a, b in fwd_ev)
    bwd_ms = statistics.mean(a.elapsed_time(b) for a, b in bwd_ev) if bwd_ev else None

    # End to end through the public API with host buffers: every step copies
    # its inputs (Q, K, V, dO) from pinned host memory and reads its results
    # (O, dQ, dK, dV) back, all inside the timed region. Steps are pipelined
    # over three streams with two device buffer sets: step i+1's uploads and
    # step i-1's downloads overlap step i's kernels.
    names = ("o", "dq", "dk", "dv") if w.bwd else ("o",)
    host_in = [t.cpu().pin_memory() for t in (q, k, v, do)]
    n_in = 4 if w.bwd else 3
    host_out = [{n: torch.empty(out[n].shape, dtype=out[n].dtype, pin_memory=True) for n in names}
                for _ in range(2)]
    dev_in = [[torch.empty_like(t) for t in (q, k, v, do)] for _ in range(2)]
    dev_out = [{n: torch.empty_like(out[n]) for n in out} for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_in[:n_in])
    d2h = sum(host_out[0][n].numel() * host_out[0][n].element_size() for n in names)
    s_h2d, s_comp, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_steps(n, start_event):
        for st in (s_h2d, s_comp, s_d2h):
            st.wait_event(start_event)
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_h2d):
                if i >= 2:
                    s_h2d.wait_event(ev_comp[b])      # dev_in[b] no longer read
                for h, d in zip(host_in[:n_in], dev_in[b][:n_in]):
                    d.copy_(h, non_blocking=True)
                ev_in[b].record(s_h2d)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_in[b])
                if i >= 2:
                    s_comp.wait_event(ev_out[b])     # dev_out[b] already read back
                step(tuple(dev_in[b]), dev_out[b])
                ev_comp[b].record(s_comp)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ev_comp[b])
                for nm in names:
                    host_out[b][nm].copy_(dev_out[b][nm], non_blocking=True)
                ev_out[b].record(s_d2h)
        return ev_out[(n - 1) % 2]

    w0 = torch.cuda.Event()
    w0.record(stream)
    last = e2e_steps(max(1, args.warmup), w0)
    stream.wait_event(last)
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    last = e2e_steps(args.steps, e0)
    stream.wait_event(last)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    return {"ms": ms, "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "clocks": clk.summary(), "e2e_ms": e2e_ms,
            "h2d": h2d, "d2h": d2h, "launches": launches_per_step * args.steps}


def cpu_sample_run(w, min_seconds=0.0):
    """The oracle as it stands on a bounded sample: the first 8000 tokens (one
    emulated rank's worth) of one head, causal fwd (+ bwd), fp64 on the host;
    further heads are added until at least ``min_seconds`` of CPU work ran."""
    import oracle
    Ls = min(8000, w.L)
    g = torch.Generator().manual_seed(0)
    heads, dt = 0, 0.0
    while heads < w.B * w.H and (heads == 0 or dt < min_seconds):
        q, k, v, do = (torch.randn(Ls, w.D, generator=g).to(w.torch_dtype).double().numpy() for _ in range(4))
        t0 = time.perf_counter()
        oracle.attention(q, k, v, w.scale, w.causal, row_block=1000)
        if w.bwd:
            oracle.attention_bwd(q, k, v, do, w.scale, w.causal, row_block=1000)
        dt += time.perf_counter() - t0
        heads += 1
    fl = heads * 4.0 * w.D * Ls * Ls * (0.5 if w.causal else 1.0) * (3.5 if w.bwd else 1.0)
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{heads} head(s) x first {Ls} tokens, {'fwd+bwd' if w.bwd else 'fwd'}, numpy fp64 "
                      f"BLAS, {dt:.2f} s"}


def blas_threads():
    """Threads the oracle's BLAS runs with (its matmuls are where the time goes)."""
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    args = ap.parse_args()
    w = WORKLOADS[args.workload]
    flops_step, fwd_flops = step_flops(w)
    config = {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "D": w.D, "cp": w.cp,
              "layout": ("contiguous", "head_tail", "striped")[w.layout], "causal": w.causal,
              "docs": len(w.docs) or None, "H_kv": w.kv_heads, "rope": ("half pairs, base %g, fused into the permute of q,k and the "
                                              "unpermute of dQ,dK" % ROPE_BASE) if w.rope else None,
              "step": "permute q,k,v" + (",dO" if w.bwd else "") + " -> ring fwd -> unpermute O" +
                      (" -> ring bwd -> unpermute dQ,dK,dV" if w.bwd else ""),
              "l2": "inputs larger than L2 (%.0f MB per tensor vs 126 MB)" % (w.B * w.H * w.L * w.D * 2 / 1e6),
              "parallelism": "replicas"}

    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return
        runs = [cpu_sample_run(w) for _ in range(args.warmup)]
        runs = [cpu_sample_run(w) for _ in range(args.steps)]
        val = statistics.median(r["value"] for r in runs)
        cb = dict(runs[0])
        cb["value"] = val
        line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
                "cpu_baseline": cb, "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                                            "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    rank, world, local = dist_setup(args.gpus)
    r = run_ours(args, w, rank, world, local)
    pk, pk_kind = peaks()
    value = aggregate_tflops(flops_step, args.steps, world, r["ms"])
    e2e_value = aggregate_tflops(flops_step, args.steps, world, r["e2e_ms"])
    # Dominant kernel: the backward when present (2.5x the forward's FLOPs).
    if w.bwd:
        kname, kflops, kms = "ring_bwd", 2.5 * fwd_flops, r["bwd_ms"]
    else:
        kname, kflops, kms = "ring_fwd", fwd_flops, r["fwd_ms"]
    sustained = pk.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    burst = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    achieved = kflops / (kms / 1e3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["ms"] / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) Q/K/V/dO)", "config": config,
        "pct_of_bf16_peak": {"burst": 100.0 * value / world / burst, "sustained": 100.0 * value / world / sustained,
                             "source": pk_kind},
        "kernels": {"ring_fwd": {"ms": r["fwd_ms"], "tflops": fwd_flops / (r["fwd_ms"] / 1e3) / 1e12},
                    "ring_bwd": ({"ms": r["bwd_ms"], "tflops": 2.5 * fwd_flops / (r["bwd_ms"] / 1e3) / 1e12}
                                 if r["bwd_ms"] else None)},
        "roofline": {"kernel": kname, "bound": "tensor", "achieved": achieved, "peak": sustained,
                     "peak_kind": f"bf16_tflops_sustained ({pk_kind}); timed inside a long step",
                     "unit": "TFLOP/s", "frac": achieved / sustained, "frac_of_burst": achieved / burst,
                     "traffic": NCU_TRAFFIC.get(w.name) if w.bwd else None},
        "clocks": r["clocks"],
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": r["launches"],
    }
    if rank == 0:
        if world == 1:
            line["cpu_baseline"] = cpu_sample_run(w, min_seconds=10.0)
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
