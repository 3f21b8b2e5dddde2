"""rattn_ring_bwd_noalloc: the ring backward for callers that cannot allocate
device memory (no allocator reachable, allocation forbidden after start-up,
or a fixed memory budget), with its scratch in the library's own fixed device
array instead of a caller workspace.

Called through the C ABI twice in a row (the shared array keeps the previous
call's contents, so the second call checks that what must start at zero is
cleared), and compared with rattn_ring_bwd, which takes a workspace, within
the gradient tolerance of the other tests. Collected last on purpose.
"""
import ctypes

import pytest
import torch

from context_ring_attention_emulated_b200.workloads import make_tensor
from tests.gpu_common import check_grad, load_rattn

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("dtype,B,H,L,D,cp,causal", [
    (torch.bfloat16, 1, 4, 2000, 128, 4, 1),
    (torch.bfloat16, 2, 2, 777, 64, 3, 1),
    (torch.float32, 1, 2, 300, 64, 2, 0),
])
def test_noalloc_matches_workspace_call_twice(dtype, B, H, L, D, cp, causal):
    rattn = load_rattn()
    lib = rattn.lib
    scale = D ** -0.5
    q, k, v, do = (make_tensor((B, H, L, D), dtype, "cuda", seed=s) for s in (51, 52, 53, 54))
    qp, pos = rattn.cp_layout_permute(q, cp)
    kp, _ = rattn.cp_layout_permute(k, cp)
    vp, _ = rattn.cp_layout_permute(v, cp)
    dop, _ = rattn.cp_layout_permute(do, cp)
    Lp = qp.shape[2]
    o, lse = rattn.rattn_ring_fwd(qp, kp, vp, pos, cp, causal=bool(causal), L_valid=L)
    ref = rattn.rattn_ring_bwd(qp, kp, vp, o, dop, lse, pos, cp, causal=bool(causal), L_valid=L)
    torch.cuda.synchronize()
    dcode = rattn.BF16 if dtype == torch.bfloat16 else rattn.F32
    for _ in range(2):
        dq, dk, dv = torch.full_like(qp, 7.0), torch.full_like(kp, 7.0), torch.full_like(vp, 7.0)
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        code = lib.rattn_ring_bwd_noalloc(_ptr(qp), _ptr(kp), _ptr(vp), _ptr(o), _ptr(dop), _ptr(lse), _ptr(pos),
                                          B, H, Lp, D, dcode, cp, 1, causal, ctypes.c_float(scale), L,
                                          _ptr(dq), _ptr(dk), _ptr(dv), stream)
        assert code == rattn.OK, rattn.status_string(code)
        torch.cuda.synchronize()
        assert rattn.rattn_get_device_error()[0] == rattn.OK
        for got, r in zip((dq, dk, dv), ref):
            check_grad(got.float().cpu().numpy(), r.float().cpu().numpy())


def test_noalloc_rejects_requests_beyond_its_array():
    rattn = load_rattn()
    lib = rattn.lib
    B, H, Lp, D = 1, 32, 32000, 128
    assert rattn.rattn_ring_bwd_workspace_size(B, H, Lp, D) > (32 << 20)
    fake = ctypes.c_void_p(0x10000)   # never dereferenced: the size check comes first
    code = lib.rattn_ring_bwd_noalloc(fake, fake, fake, fake, fake, fake, fake, B, H, Lp, D, rattn.BF16, 4, 1, 1,
                                      ctypes.c_float(0.088), Lp, fake, fake, fake, None)
    assert code == rattn.ERR_UNSUPPORTED
