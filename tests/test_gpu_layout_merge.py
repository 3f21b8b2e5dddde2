"""GPU parity: layout permute/unpermute (bit-exact against the oracle's index
map, positions included) and the standalone online-softmax merge."""
import numpy as np
import pytest
import torch

import oracle
from context_ring_attention_emulated_b200.workloads import WORKLOADS, make_tensor
from tests.gpu_common import TOL_F32, load_rattn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rattn():
    return load_rattn()


def _bits(t):
    return t.view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32).cpu().numpy()


@pytest.mark.parametrize("dtype,D", [(torch.float32, 64), (torch.bfloat16, 128), (torch.bfloat16, 8),
                                     (torch.float32, 4)])
@pytest.mark.parametrize("L,cp,layout", [(256, 2, 1), (4096, 2, 1), (29, 3, 1), (29, 3, 0), (1000, 4, 1),
                                         (7, 8, 1), (1, 1, 1), (130, 16, 1), (97, 5, 0), (29, 3, 2),
                                         (1000, 4, 2), (7, 8, 2), (130, 16, 2), (4096, 2, 2)])
def test_permute_unpermute_bit_exact(rattn, dtype, D, L, cp, layout):
    x = make_tensor((2, 3, L, D), dtype, "cuda", seed=L + cp)
    y, pos = rattn.cp_layout_permute(x, cp, layout)
    Lp, src, pos_ref = oracle.perm_index(L, cp, layout)
    assert y.shape[2] == Lp
    assert np.array_equal(pos.cpu().numpy(), pos_ref)
    y_ref, _ = oracle.permute(_bits(x), cp, layout)
    assert np.array_equal(_bits(y), y_ref)
    back = rattn.cp_layout_unpermute(y, L, cp, layout)
    assert np.array_equal(_bits(back), _bits(x))


@pytest.mark.parametrize("name", ["bf16_L32000_cp4", "bf16_L1M_cp8", "bf16_L131072_cp8_noncausal",
                                  "bf16_L32000_cp4_striped"])
def test_permute_full_size(rattn, name):
    w = WORKLOADS[name]
    x = make_tensor((w.B, w.H, w.L, w.D), w.torch_dtype, "cuda", seed=3)
    y, pos = rattn.cp_layout_permute(x, w.cp, w.layout)
    Lp, src, pos_ref = oracle.perm_index(w.L, w.cp, w.layout)
    assert np.array_equal(pos.cpu().numpy(), pos_ref)
    xb = x.view(torch.int16).cpu()
    yb = y.view(torch.int16).cpu()
    assert torch.equal(yb, xb[:, :, torch.from_numpy(src)])        # no padding at these sizes
    back = rattn.cp_layout_unpermute(y, w.L, w.cp, w.layout)
    assert torch.equal(back.view(torch.int16).cpu(), xb)


def _lse_case(shape, seed):
    g = np.random.default_rng(seed)
    a = g.standard_normal(shape) * 4
    b = g.standard_normal(shape) * 4
    a[..., ::7] = -np.inf            # accumulator empty
    b[..., ::5] = -np.inf            # block empty
    return a, b


@pytest.mark.parametrize("D", [64, 128, 12])
def test_merge_matches_oracle(rattn, D):
    B, H, Lq = 2, 3, 333
    g = np.random.default_rng(D)
    oa, ob = g.standard_normal((B, H, Lq, D)), g.standard_normal((B, H, Lq, D))
    la, lb = _lse_case((B, H, Lq), D)
    oa[np.isneginf(la)] = 0.0
    ob[np.isneginf(lb)] = 0.0
    o_ref, l_ref = oracle.merge(oa, la, ob, lb)
    t = lambda a: torch.tensor(a, dtype=torch.float32, device="cuda")
    o_acc, l_acc = t(oa), t(la)
    rattn.rattn_merge(o_acc, l_acc, t(ob), t(lb))
    got_l = l_acc.cpu().double().numpy()
    assert np.array_equal(np.isneginf(got_l), np.isneginf(l_ref))
    fin = np.isfinite(l_ref)
    assert np.abs(got_l[fin] - l_ref[fin]).max() <= TOL_F32
    assert np.abs(o_acc.cpu().double().numpy() - o_ref).max() <= TOL_F32
    assert not torch.isnan(o_acc).any()
