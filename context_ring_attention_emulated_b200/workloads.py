"""Seeded synthetic workloads shaped like the pages' examples.

This module holds input generation only (no attention arithmetic). Both the
CUDA path's tests/bench and the oracle consume what it produces.

Shapes follow the pages: the 2-rank example of the Ultralytics glossary
"Context Parallelism" (B=1, H=4, L=4096, D=64, bf16, causal, seed 0), the
32,000-token / 4-way split of the same page's "How context parallelism works",
and the 1M-token / 8-GPU use case of "Sequence parallelism and ring attention"
("Real implementations"). Q, K, V are drawn in that order from one generator
as float32 standard normals (times ``mult``), then rounded to the dtype.
"""
from dataclasses import dataclass

import torch

LAYOUT_CONTIGUOUS = 0
LAYOUT_HEAD_TAIL = 1
LAYOUT_STRIPED = 2


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str          # "f32" or "bf16"
    B: int
    H: int
    L: int
    D: int
    causal: bool
    cp: int
    layout: int
    mult: float = 1.0
    bwd: bool = False
    H_kv: int = 0       # key/value heads (grouped-query attention); 0 means H
    rope: bool = False  # rotate Q and K at their global positions while permuting
    docs: tuple = ()    # packed sequences: document lengths summing to L (empty: one sequence)

    @property
    def kv_heads(self):
        return self.H_kv or self.H

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def scale(self):
        return self.D ** -0.5

    def causal_flops_fwd(self):
        """Algorithmic forward FLOPs: 4*B*H*D*L^2, halved when causal; for a
        pack of documents the sum of L_i^2 over the documents replaces L^2."""
        sq = sum(d * d for d in self.docs) if self.docs else self.L * self.L
        f = 4.0 * self.B * self.H * self.D * sq
        return f / 2 if self.causal else f

    @property
    def cu_seqlens(self):
        out = [0]
        for d in self.docs:
            out.append(out[-1] + d)
        return out


def doc_lengths(total, n, lo, hi, seed):
    """Seeded document lengths for a pack: n - 1 lengths drawn uniformly from
    [lo, hi), the last one taking the rest of ``total`` (the draws are cut
    short if they already reach it)."""
    g = torch.Generator().manual_seed(seed)
    out = []
    for _ in range(n - 1):
        d = int(torch.randint(lo, hi, (1,), generator=g).item())
        if sum(out) + d >= total:
            break
        out.append(d)
    out.append(total - sum(out))
    return tuple(out)


WORKLOADS = {
    "fp32_L256_cp2": Workload("fp32_L256_cp2", "f32", 1, 2, 256, 64, True, 2, LAYOUT_HEAD_TAIL),
    "bf16_L4096_cp2": Workload("bf16_L4096_cp2", "bf16", 1, 4, 4096, 64, True, 2, LAYOUT_HEAD_TAIL),
    "bf16_L32000_cp4": Workload("bf16_L32000_cp4", "bf16", 1, 32, 32000, 128, True, 4, LAYOUT_HEAD_TAIL),
    "bf16_L1M_cp8": Workload("bf16_L1M_cp8", "bf16", 1, 8, 1048576, 128, True, 8, LAYOUT_HEAD_TAIL, 0.5),
    "bf16_L131072_cp8_noncausal": Workload("bf16_L131072_cp8_noncausal", "bf16", 1, 8, 131072, 128, False, 8,
                                           LAYOUT_CONTIGUOUS, 0.5),
    "bf16_L32000_cp4_fwdbwd": Workload("bf16_L32000_cp4_fwdbwd", "bf16", 1, 32, 32000, 128, True, 4,
                                       LAYOUT_HEAD_TAIL, 1.0, True),
    # The 32k / cp=4 shapes under the striped assignment (token g on rank g mod cp).
    "bf16_L32000_cp4_striped": Workload("bf16_L32000_cp4_striped", "bf16", 1, 32, 32000, 128, True, 4,
                                        LAYOUT_STRIPED),
    "bf16_L32000_cp4_striped_fwdbwd": Workload("bf16_L32000_cp4_striped_fwdbwd", "bf16", 1, 32, 32000, 128, True,
                                               4, LAYOUT_STRIPED, 1.0, True),
    # The 32k / cp=4 step with 8 key/value heads shared by 32 query heads (GQA).
    "bf16_L32000_cp4_gqa8_fwdbwd": Workload("bf16_L32000_cp4_gqa8_fwdbwd", "bf16", 1, 32, 32000, 128, True, 4,
                                            LAYOUT_HEAD_TAIL, 1.0, True, H_kv=8),
    # A 32,000-token pack of 24 documents (23 drawn from 64..2599 tokens, the last
    # taking the rest) laid out per
    # document (packed sequences), cp=4 head-tail, causal within documents.
    "bf16_L32000_cp4_varlen_fwdbwd": Workload("bf16_L32000_cp4_varlen_fwdbwd", "bf16", 1, 32, 32000, 128, True, 4,
                                              LAYOUT_HEAD_TAIL, 1.0, True, docs=doc_lengths(32000, 24, 64, 2600, 7)),
    # The 32k / cp=4 step with RoPE fused into the permute of Q, K and the
    # unpermute of dQ, dK.
    "bf16_L32000_cp4_rope_fwdbwd": Workload("bf16_L32000_cp4_rope_fwdbwd", "bf16", 1, 32, 32000, 128, True, 4,
                                            LAYOUT_HEAD_TAIL, 1.0, True, rope=True),
}


def make_qkv(w: Workload, device="cpu", seed=0):
    """Q [B, H, L, D] and K, V [B, H_kv, L, D] in the workload's dtype, from
    one seeded generator."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = []
    for heads in (w.H, w.kv_heads, w.kv_heads):
        x = torch.randn(w.B, heads, w.L, w.D, generator=g, device=device, dtype=torch.float32)
        if w.mult != 1.0:
            x.mul_(w.mult)
        out.append(x.to(w.torch_dtype))
    return out


def make_unit_grad(w: Workload, device="cpu", seed=1):
    """An upstream gradient dO ~ N(0, 1) [B, H, L, D] in the workload's dtype."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn(w.B, w.H, w.L, w.D, generator=g, device=device, dtype=torch.float32).to(w.torch_dtype)


def make_tensor(shape, dtype, device="cpu", seed=0, mult=1.0):
    """Generic seeded standard-normal tensor (float32 draw, then cast)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if mult != 1.0:
        x.mul_(mult)
    return x.to(dtype)
