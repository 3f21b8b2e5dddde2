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
import glob
import hashlib
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
# Packed workloads pad every document's share of a rank slice to whole
# 128-row tiles, so that no kernel tile straddles two documents.
VARLEN_ALIGN = 128
# DRAM bytes (read + write) per launch of the dominant kernel from one ncu
# capture (dram__bytes_read.sum + dram__bytes_write.sum) of the kernel as it
# stands, taken on a smaller case and scaled to the workload's launch by the
# sequence length. Empty while the kernel has changed since its last capture.
# The ring backward at B=1 H=32 L=16000 D=128 cp=4: 791,380,480 B read +
# 477,255,936 B written, x2 for L=32000; algorithmic 2,621,440,000 B (Q, K, V,
# dO read, the fp32 dQ accumulator read and written, dK and dV written).
NCU_TRAFFIC = {"bf16_L32000_cp4_fwdbwd": {"bytes": 2 * (791380480 + 477255936),
                                          "ratio": 2 * (791380480 + 477255936) / 2621440000}}
# Dense bf16 tensor rate of one SM: a 128x128x16 MMA every 64 cycles.
SM_COUNT = 148
TENSOR_FLOP_PER_CLK_SM = 8192


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
                                          "--format=csv,noheader,nounits", "-lms", "50"],
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
        plan = rattn.cp_layout_varlen_plan(w.cu_seqlens, cp, layout, VARLEN_ALIGN)
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
    # Rows 0..Ls-1 of the first heads, inputs and results of the last timed
    # step: under a causal mask they depend on nothing past row Ls, so the
    # oracle can recompute them from this prefix alone.
    sample = None
    if w.causal and not w.docs and Hkv == H:
        Ls, nh = min(8000, L), min(8, B * H)
        pick = lambda t: t.reshape(B * H, L, D)[:nh, :Ls].float().cpu()
        sample = {"q": pick(q), "k": pick(k), "v": pick(v), "do": pick(do), "o": pick(out["o"]),
                  "dq": pick(out["dq"]) if w.bwd else None, "rows": Ls}
    return {"ms": ms, "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "clocks": clk.summary(), "e2e_ms": e2e_ms,
            "h2d": h2d, "d2h": d2h, "launches": launches_per_step * args.steps, "sample": sample}


def median_event_ms(fn, reps, warmup, stream):
    """Median CUDA-event time of ``fn`` on ``stream`` over ``reps`` calls after
    ``warmup`` untimed ones."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    evs = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in evs)


def tensor_rate_at(sm_mhz):
    """Dense bf16 tensor-core FLOP/s of the whole GPU at an SM clock (MHz)."""
    return SM_COUNT * TENSOR_FLOP_PER_CLK_SM * sm_mhz * 1e6 if sm_mhz else None


def extra_measurements(local, pk):
    """Kernels the default step does not time, each measured on its own after
    the step's timed regions: the 1M-token causal ring forward (8 heads, cp=8
    head-tail), and the bandwidth kernels (merge, permute, unpermute) at the
    32k and 1M sizes. Inputs are larger than L2 in every case."""
    from context_ring_attention_emulated_b200 import rattn
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    burst = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    hbm = pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    res = {}

    w = WORKLOADS["bf16_L1M_cp8"]
    q, k, v = make_qkv(w, dev, seed=0)
    Lp = rattn.cp_layout_padded_len(w.L, w.cp, w.layout)
    qp, pos = rattn.cp_layout_permute(q, w.cp, w.layout)
    kp, _ = rattn.cp_layout_permute(k, w.cp, w.layout)
    vp, _ = rattn.cp_layout_permute(v, w.cp, w.layout)
    o = torch.empty_like(qp)
    lse = torch.empty(w.B, w.H, Lp, dtype=torch.float32, device=dev)
    fwd = lambda: rattn.rattn_ring_fwd(qp, kp, vp, pos, w.cp, w.layout, True, w.scale, L_valid=w.L, o=o, lse=lse)
    with ClockSampler(local) as clk:
        ms = median_event_ms(fwd, 3, 1, stream)
    c = clk.summary()
    tf = w.causal_flops_fwd() / (ms / 1e3) / 1e12
    at_clk = tensor_rate_at(c["sm_mhz"])
    res["ring_fwd_" + w.name] = {"ms": ms, "tflops": tf, "frac_of_burst": tf / burst,
                                 "frac_at_clock": tf * 1e12 / at_clk if at_clk else None, "clocks": c,
                                 "reps": "median of 3 after 1 warm-up"}

    def bw_entry(name, fn, nbytes, reps=10):
        ms_ = median_event_ms(fn, reps, 3, stream)
        gbs = nbytes / (ms_ / 1e3) / 1e9
        res[name] = {"ms": ms_, "GB_per_s": gbs, "frac_of_hbm": gbs / hbm, "bytes": nbytes}

    es = 2
    n1m = w.B * w.H * w.L * w.D * es
    bw_entry("permute_" + w.name, lambda: rattn.cp_layout_permute(q, w.cp, w.layout, y=qp, pos=pos), 2 * n1m + 4 * Lp)
    bw_entry("unpermute_" + w.name, lambda: rattn.cp_layout_unpermute(qp, w.L, w.cp, w.layout, x=q), 2 * n1m)
    del q, k, v, qp, kp, vp, o, lse, pos
    torch.cuda.empty_cache()

    w = WORKLOADS["bf16_L32000_cp4"]
    x = make_qkv(w, dev, seed=0)[0]
    Lp = rattn.cp_layout_padded_len(w.L, w.cp, w.layout)
    y = torch.empty(w.B, w.H, Lp, w.D, dtype=x.dtype, device=dev)
    pos = torch.empty(Lp, dtype=torch.int32, device=dev)
    n32 = w.B * w.H * w.L * w.D * es
    bw_entry("permute_" + w.name, lambda: rattn.cp_layout_permute(x, w.cp, w.layout, y=y, pos=pos), 2 * n32 + 4 * Lp)
    bw_entry("unpermute_" + w.name, lambda: rattn.cp_layout_unpermute(y, w.L, w.cp, w.layout, x=x), 2 * n32)
    rows = w.B * w.H * w.L
    o_acc = torch.randn(w.B, w.H, w.L, w.D, device=dev)
    o_blk = torch.randn(w.B, w.H, w.L, w.D, device=dev)
    l_acc = torch.randn(w.B, w.H, w.L, device=dev)
    l_blk = torch.randn(w.B, w.H, w.L, device=dev)
    bw_entry("merge_" + w.name, lambda: rattn.rattn_merge(o_acc, l_acc, o_blk, l_blk), rows * (12 * w.D + 12))
    err, site = rattn.rattn_get_device_error()
    if err != rattn.OK:
        raise RuntimeError(f"device-side wait timed out at site {site}")
    return res


def source_digest():
    """Commit of the checkout when git can tell, and a digest of the library
    sources and this file (which identifies the code when no .git travels)."""
    sha = None
    try:
        r = subprocess.run(["git", "rev-parse", "HEAD"], cwd=ROOT, capture_output=True, text=True, timeout=10)
        if r.returncode == 0:
            sha = r.stdout.strip()
    except (OSError, subprocess.SubprocessError):
        pass
    h = hashlib.sha256()
    pkg = os.path.join(ROOT, "context_ring_attention_emulated_b200")
    files = sorted(glob.glob(os.path.join(pkg, "csrc", "*")) + glob.glob(os.path.join(ROOT, "include", "*.h")) +
                   [os.path.join(pkg, "rattn.py"), os.path.abspath(__file__)])
    for f in files:
        h.update(os.path.relpath(f, ROOT).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return {"git": sha, "src_sha256": h.hexdigest()[:16]}


def cpu_sample_run(w, min_seconds=0.0, sample=None):
    """The oracle as it stands on a bounded sample: the first 8000 tokens (one
    emulated rank's worth) of one head, causal fwd (+ bwd), fp64 on the host;
    further heads are added until at least ``min_seconds`` of CPU work ran.

    With ``sample`` (rows 0..Ls-1 of the first heads of the GPU run: inputs,
    O and dQ), the oracle runs on exactly those inputs, and the GPU's O and dQ
    on those rows are compared with its results (a causal prefix depends on
    nothing after it), giving the line a parity record."""
    import numpy as np

    import oracle
    Ls = sample["rows"] if sample else min(8000, w.L)
    n_avail = sample["q"].shape[0] if sample else w.B * w.H
    g = torch.Generator().manual_seed(0)
    heads, dt = 0, 0.0
    err = {"o_max_abs": 0.0, "o_viol": 0, "dq_max_abs": 0.0, "dq_ref_max": 0.0}
    while heads < n_avail and (heads == 0 or dt < min_seconds):
        if sample:
            q, k, v, do = (sample[n][heads].double().numpy() for n in ("q", "k", "v", "do"))
        else:
            q, k, v, do = (torch.randn(Ls, w.D, generator=g).to(w.torch_dtype).double().numpy() for _ in range(4))
        t0 = time.perf_counter()
        o_ref, _ = oracle.attention(q, k, v, w.scale, w.causal, row_block=1000)
        grads = oracle.attention_bwd(q, k, v, do, w.scale, w.causal, row_block=1000) if w.bwd else None
        dt += time.perf_counter() - t0
        if sample:
            e = np.abs(sample["o"][heads].double().numpy() - o_ref)
            err["o_max_abs"] = max(err["o_max_abs"], float(e.max()))
            err["o_viol"] += int((e > 2e-2 + 1e-2 * np.abs(o_ref)).sum())
            if grads is not None and sample["dq"] is not None:
                err["dq_max_abs"] = max(err["dq_max_abs"],
                                        float(np.abs(sample["dq"][heads].double().numpy() - grads[0]).max()))
                err["dq_ref_max"] = max(err["dq_ref_max"], float(np.abs(grads[0]).max()))
        heads += 1
    fl = heads * 4.0 * w.D * Ls * Ls * (0.5 if w.causal else 1.0) * (3.5 if w.bwd else 1.0)
    out = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
           "sample": f"{heads} head(s) x first {Ls} tokens{' of the GPU run' if sample else ''}, "
                     f"{'fwd+bwd' if w.bwd else 'fwd'}, numpy fp64 BLAS, {dt:.2f} s"}
    if sample:
        par = {"rows": f"heads 0..{heads - 1}, global rows 0..{Ls - 1} of the last timed step",
               "o_max_abs": err["o_max_abs"], "o_elements_outside_tol": err["o_viol"],
               "tolerance": "O: |x-ref| <= 2e-2 + 1e-2|ref|; dQ: 3e-2 max-abs"}
        if w.bwd:
            par["dq_max_abs"] = err["dq_max_abs"]
            par["dq_max_abs_over_ref_max"] = err["dq_max_abs"] / err["dq_ref_max"] if err["dq_ref_max"] else None
        par["pass"] = err["o_viol"] == 0 and (not w.bwd or err["dq_max_abs"] <= 3e-2)
        out["parity"] = par
    return out


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
    ap.add_argument("--no-extra", action="store_true", help="skip the per-kernel measurements after the step")
    args = ap.parse_args()
    w = WORKLOADS[args.workload]
    flops_step, fwd_flops = step_flops(w)
    config = {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "D": w.D, "cp": w.cp,
              "layout": ("contiguous", "head_tail", "striped")[w.layout], "causal": w.causal,
              "docs": len(w.docs) or None,
              "varlen_align": VARLEN_ALIGN if w.docs else None, "H_kv": w.kv_heads, "rope": ("half pairs, base %g, fused into the permute of q,k and the "
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
                "steps": args.steps, "warmup": args.warmup,
                # the whole step's FLOPs at the sampled rate (the oracle runs a bounded sample of it)
                "ms_per_step": flops_step / (val * 1e12) * 1e3, "ms_per_step_kind": "extrapolated from the sample",
                "higher_is_better": True, "scaling": "weak",
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
    at_clk = tensor_rate_at(r["clocks"]["sm_mhz"])
    traffic = NCU_TRAFFIC.get(w.name) if w.bwd else None
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["ms"] / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) Q/K/V/dO)", "config": config,
        "pct_of_bf16_peak": {"burst": 100.0 * value / world / burst, "sustained": 100.0 * value / world / sustained,
                             "source": pk_kind},
        "kernels": {"ring_fwd": {"ms": r["fwd_ms"], "tflops": fwd_flops / (r["fwd_ms"] / 1e3) / 1e12},
                    "ring_bwd": ({"ms": r["bwd_ms"], "tflops": 2.5 * fwd_flops / (r["bwd_ms"] / 1e3) / 1e12}
                                 if r["bwd_ms"] else None)},
        "roofline": {"kernel": kname, "bound": "tensor", "achieved": achieved, "peak": burst,
                     "peak_kind": f"bf16_tflops burst ({pk_kind})", "unit": "TFLOP/s", "frac": achieved / burst,
                     "frac_of_sustained": achieved / sustained,
                     "tensor_rate_at_clock": at_clk / 1e12 if at_clk else None,
                     "frac_at_clock": achieved * 1e12 / at_clk if at_clk else None,
                     "traffic": traffic["bytes"] if traffic else None,
                     "traffic_over_algorithmic": traffic["ratio"] if traffic else None},
        "clocks": r["clocks"],
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": r["launches"],
        "source": source_digest(),
    }
    if rank == 0 and world == 1:
        if not args.no_extra and w.name == DEFAULT:
            line["extra"] = extra_measurements(local, pk)
        line["cpu_baseline"] = cpu_sample_run(w, min_seconds=10.0, sample=r["sample"])
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
