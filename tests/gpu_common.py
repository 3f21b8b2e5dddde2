"""Shared helpers for the GPU parity tests: library loading, oracle calls on
the same seeded inputs, and the tolerance checks the targets state.

Tolerances (elementwise, written here once):
  fp32 path:  |x - ref| <= 1e-4 on O and LSE
  bf16 path:  O: |x - ref| <= 2e-2 + 1e-2 |ref|;  LSE: |x - ref| <= 1e-3;
              gradients: |g - ref| <= 3e-2, plus a scale-free check
              max|g - ref| <= 3e-2 max|ref|.
Permutation, positions and layout copies: bit-exact.
"""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402

TOL_F32 = 1e-4
TOL_BF16_O_ABS, TOL_BF16_O_REL = 2e-2, 1e-2
TOL_BF16_LSE = 1e-3
TOL_GRAD = 3e-2


def load_rattn():
    from context_ring_attention_emulated_b200 import build as b
    b.build(debug=os.environ.get("RATTN_DEBUG", "0") == "1")
    from context_ring_attention_emulated_b200 import rattn
    return rattn


def to64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def check_o(got, ref, dtype):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    err = np.abs(got - ref)
    if dtype == torch.float32:
        assert err.max() <= TOL_F32, f"max abs err {err.max():.3e} > {TOL_F32}"
    else:
        bound = TOL_BF16_O_ABS + TOL_BF16_O_REL * np.abs(ref)
        bad = err > bound
        assert not bad.any(), f"{bad.sum()} elements out of tolerance; max abs err {err.max():.3e}"
    return float(err.max())


def check_lse(got, ref, dtype):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.array_equal(np.isneginf(got), np.isneginf(ref)), "-inf pattern differs"
    fin = np.isfinite(ref)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16_LSE
    err = np.abs(got[fin] - ref[fin]) if fin.any() else np.zeros(1)
    assert err.max() <= tol, f"LSE max abs err {err.max():.3e} > {tol}"
    return float(err.max())


def check_grad(got, ref, scale_free=True):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    assert err.max() <= TOL_GRAD, f"grad max abs err {err.max():.3e}"
    if scale_free and np.abs(ref).max() > 0:
        rel = err.max() / np.abs(ref).max()
        assert rel <= TOL_GRAD, f"grad normalised err {rel:.3e}"
    return float(err.max())


def oracle_ring_reference(q, k, v, cp, layout, causal, scale):
    """Oracle answer for the ring forward in rank-major order: full attention
    on the global sequence, then permuted (pad rows excluded by the caller)."""
    L = q.shape[-2]
    o, lse = oracle.attention(to64(q), to64(k), to64(v), scale, causal)
    op, pos = oracle.permute(o, cp, layout)
    lp, _ = oracle.permute(lse[..., None], cp, layout)
    return op, lp[..., 0], pos, L
