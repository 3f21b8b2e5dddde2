"""GPU parity of the RoPE-fused layout calls against the fp64 oracle.

cp_layout_permute_rope must equal the oracle's rotation at the global
positions followed by the layout permute; cp_layout_unpermute_rope_grad must
equal the oracle's inverse rotation of the unpermuted gradient. Every layout,
both pairings, padding, positions up to 2^20, and the whole path (RoPE on
Q and K, ring forward and backward, gradients back through the rotation).

Tolerance of the rotated values (written here once): the kernel forms the
angle in fp64 and reduces it modulo 2 pi there, takes sin/cos and rotates in
fp32 and rounds once to the dtype, so
  bf16: |x - ref| <= 2^-8 |ref| + 1e-5     (one rounding of the exact value,
                                             with a factor 2 of slack)
  fp32: |x - ref| <= 1e-6 |ref| + 1e-5
Positions and pad rows: bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle
from context_ring_attention_emulated_b200.workloads import WORKLOADS, make_tensor
from tests.gpu_common import check_grad, check_lse, check_o, load_rattn, to64

pytestmark = pytest.mark.gpu

HALF, INTERLEAVED = oracle.ROPE_HALF, oracle.ROPE_INTERLEAVED


@pytest.fixture(scope="module")
def rattn():
    return load_rattn()


def check_rot(got, ref, dtype):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    rtol = 2.0 ** -8 if dtype == torch.bfloat16 else 1e-6
    bad = np.abs(got - ref) > rtol * np.abs(ref) + 1e-5
    assert not bad.any(), f"{bad.sum()} of {bad.size} out of tolerance; max err {np.abs(got - ref).max():.3e}"


CASES = [
    # dtype, D, L, cp, layout
    (torch.bfloat16, 128, 1000, 4, 1),
    (torch.bfloat16, 64, 29, 4, 1),        # padded to 32
    (torch.bfloat16, 16, 97, 3, 2),        # smallest bf16 HALF row, striped, padded
    (torch.bfloat16, 128, 300, 2, 0),
    (torch.float32, 64, 256, 2, 1),
    (torch.float32, 8, 130, 16, 1),        # smallest fp32 HALF row, heavy padding
    (torch.float32, 128, 77, 5, 2),
]


@pytest.mark.parametrize("style", [HALF, INTERLEAVED])
@pytest.mark.parametrize("case", CASES)
def test_permute_rope_matches_oracle(rattn, case, style):
    dtype, D, L, cp, layout = case
    base = 10000.0 if D != 64 else 500000.0
    x = make_tensor((2, 3, L, D), dtype, "cuda", seed=L + D)
    y, pos = rattn.cp_layout_permute_rope(x, cp, layout, base, style)
    torch.cuda.synchronize()
    Lp, src, pos_ref = oracle.perm_index(L, cp, layout)
    assert np.array_equal(pos.cpu().numpy(), pos_ref)
    ref, _ = oracle.permute(oracle.rope(to64(x), np.arange(L), base, style), cp, layout)
    real = pos_ref < L
    check_rot(y.float().cpu().numpy()[..., real, :], ref[..., real, :], dtype)
    assert torch.count_nonzero(y[..., torch.from_numpy(~real).cuda(), :]).item() == 0


@pytest.mark.parametrize("style", [HALF, INTERLEAVED])
@pytest.mark.parametrize("case", CASES)
def test_unpermute_rope_grad_matches_oracle(rattn, case, style):
    dtype, D, L, cp, layout = case
    Lp = rattn.cp_layout_padded_len(L, cp, layout)
    dy = make_tensor((2, 3, Lp, D), dtype, "cuda", seed=Lp + 7)
    dx = rattn.cp_layout_unpermute_rope_grad(dy, L, cp, layout, 10000.0, style)
    torch.cuda.synchronize()
    ref = oracle.rope_grad(oracle.unpermute(to64(dy), L, cp, layout), np.arange(L), 10000.0, style)
    check_rot(dx.float().cpu().numpy(), ref, dtype)


def test_permute_rope_position_zero_and_round_trip(rattn):
    """Position 0 is not rotated (bit-exact copy), and the gradient unpermute
    undoes the rotation up to the two roundings. The rounding of a rotated
    pair is relative to the pair's length, so the bound is too:
    |back - x| <= 2^-7 |(x_i, x_{i+D/2})| + 1e-5."""
    x = make_tensor((1, 4, 4096, 128), torch.bfloat16, "cuda", seed=5)
    xf = x.float()
    pair = torch.sqrt(xf[..., :64] ** 2 + xf[..., 64:] ** 2).repeat(1, 1, 1, 2)
    for layout in (0, 1, 2):
        y, pos = rattn.cp_layout_permute_rope(x, 2, layout)
        slot0 = int(np.argmax(pos.cpu().numpy() == 0))
        assert torch.equal(y[:, :, slot0], x[:, :, 0])
        back = rattn.cp_layout_unpermute_rope_grad(y, 4096, 2, layout)
        err = (back.float() - xf).abs()
        assert (err <= 2.0 ** -7 * pair + 1e-5).all()


def test_permute_rope_full_size_1m_positions(rattn):
    """1M tokens / cp=8 head-tail (positions up to 2^20 - 1), sampled rows of
    every head against the oracle."""
    w = WORKLOADS["bf16_L1M_cp8"]
    x = make_tensor((w.B, w.H, w.L, w.D), w.torch_dtype, "cuda", seed=9, mult=w.mult)
    y, pos = rattn.cp_layout_permute_rope(x, w.cp, w.layout, 500000.0, HALF)
    torch.cuda.synchronize()
    g = np.random.default_rng(0)
    rows = np.unique(np.concatenate([g.integers(0, w.L, 256), [0, 1, w.L - 2, w.L - 1], 65536 * np.arange(16)]))
    Lp, src, pos_ref = oracle.perm_index(w.L, w.cp, w.layout)
    slot_of = np.argsort(pos_ref)
    ref = oracle.rope(to64(x[0][:, torch.from_numpy(rows).cuda()]), rows, 500000.0, HALF)
    got = y[0][:, torch.from_numpy(slot_of[rows]).cuda()].float().cpu().numpy()
    check_rot(got, ref, w.torch_dtype)


@pytest.mark.parametrize("layout,style", [(1, HALF), (2, INTERLEAVED)])
def test_rope_through_ring_fwd_bwd(rattn, layout, style):
    """The whole path with RoPE: rotate Q and K at their global positions
    while permuting, ring forward and backward, gradients of Q and K back
    through the rotation while unpermuting; against the oracle's
    attention(rope(Q), rope(K), V) and its gradient chained through rope."""
    B, H, L, D, cp = 1, 2, 1000, 128, 4
    base = 10000.0
    scale = D ** -0.5
    q, k, v = (make_tensor((B, H, L, D), torch.bfloat16, "cuda", seed=s) for s in (51, 52, 53))
    do = make_tensor((B, H, L, D), torch.bfloat16, "cuda", seed=54)
    qp, pos = rattn.cp_layout_permute_rope(q, cp, layout, base, style)
    kp, _ = rattn.cp_layout_permute_rope(k, cp, layout, base, style)
    vp, _ = rattn.cp_layout_permute(v, cp, layout)
    dop, _ = rattn.cp_layout_permute(do, cp, layout)
    o, lse = rattn.rattn_ring_fwd(qp, kp, vp, pos, cp, layout, True, scale, L_valid=L)
    dqp, dkp, dvp = rattn.rattn_ring_bwd(qp, kp, vp, o, dop, lse, pos, cp, layout, True, scale, L_valid=L)
    out = rattn.cp_layout_unpermute(o, L, cp, layout)
    dq = rattn.cp_layout_unpermute_rope_grad(dqp, L, cp, layout, base, style)
    dk = rattn.cp_layout_unpermute_rope_grad(dkp, L, cp, layout, base, style)
    dv = rattn.cp_layout_unpermute(dvp, L, cp, layout)
    torch.cuda.synchronize()
    t = np.arange(L)
    # the attention consumes the rotated Q and K as bf16 tensors: the exact
    # rotation rounded once (RNE), as the rotated values the kernel hands on
    bf = lambda a: torch.from_numpy(a).to(torch.bfloat16).double().numpy()
    qr, kr = bf(oracle.rope(to64(q), t, base, style)), bf(oracle.rope(to64(k), t, base, style))
    o_ref, l_ref = oracle.attention(qr, kr, to64(v), scale, True)
    check_o(out.float().cpu().numpy(), o_ref, torch.bfloat16)
    real = pos.cpu().numpy() < L
    l_ref_p, _ = oracle.permute(l_ref[..., None], cp, layout)
    check_lse(lse.cpu().numpy()[..., real], l_ref_p[..., 0][..., real], torch.bfloat16)
    dqr, dkr, dv_ref = oracle.attention_bwd(qr, kr, to64(v), to64(do), scale, True)
    check_grad(dq.float().cpu().numpy(), oracle.rope_grad(dqr, t, base, style))
    check_grad(dk.float().cpu().numpy(), oracle.rope_grad(dkr, t, base, style))
    check_grad(dv.float().cpu().numpy(), dv_ref)
