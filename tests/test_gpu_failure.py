"""Failure detection without a GPU fault: with the bounded-wait limit forced to
1 ns every tensor-core wait gives up at once; the kernel records the error,
drains its own in-flight copies and MMAs, frees TMEM and returns. The host
reads RATTN_ERR_TIMEOUT, and the context stays usable (a normal run after it
still matches the oracle)."""
import pytest
import torch

import oracle
from context_ring_attention_emulated_b200.workloads import make_tensor
from tests.gpu_common import check_o, load_rattn, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rattn():
    return load_rattn()


def test_forced_wait_timeout_is_reported_and_recoverable(rattn):
    B, H, L, D, cp = 1, 2, 1024, 128, 2
    q, k, v = (make_tensor((B, H, L, D), torch.bfloat16, "cuda", seed=s) for s in (41, 42, 43))
    qp, pos = rattn.cp_layout_permute(q, cp)
    kp, _ = rattn.cp_layout_permute(k, cp)
    vp, _ = rattn.cp_layout_permute(v, cp)
    torch.cuda.synchronize()
    assert rattn.rattn_get_device_error()[0] == rattn.OK
    try:
        rattn.rattn_set_wait_limit_ns(1)
        rattn.rattn_ring_fwd(qp, kp, vp, pos, cp)
        torch.cuda.synchronize()
        code, site = rattn.rattn_get_device_error()
    finally:
        rattn.rattn_set_wait_limit_ns(0)
    assert code == rattn.ERR_TIMEOUT and site > 0
    assert rattn.rattn_get_device_error()[0] == rattn.OK          # cleared
    o, _ = rattn.rattn_ring_fwd(qp, kp, vp, pos, cp)
    out = rattn.cp_layout_unpermute(o, L, cp)
    torch.cuda.synchronize()
    assert rattn.rattn_get_device_error()[0] == rattn.OK
    o_ref, _ = oracle.attention(to64(q), to64(k), to64(v), D ** -0.5, True)
    check_o(out.float().cpu().numpy(), o_ref, torch.bfloat16)
