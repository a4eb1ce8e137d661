"""Failure detection without a GPU fault: one CTA of the fused decode FFN
kernel is made to wait for 16 bytes more than its weight copies deliver (a
transaction count that can never complete).  Its wait is bounded, so it
gives up, the kernel finishes (the data it needed did arrive), the status
word reports the timeout, the results are still right, and the context stays
usable: the next call is clean."""
import time

import pytest
import torch

from gpu_helpers import ORDER_REL, rule13, workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import quantized_moe_q4_b200 as m  # noqa: E402


def test_decode_wait_timeout_reported_and_recovered():
    x, lw = workload("decode_t1", T=1000)
    L = m.Layer.from_host(lw)
    xt = torch.from_numpy(x[3:4].copy()).cuda()
    ws = m.alloc_workspace(m.moe_q4_ffn_workspace_bytes(L, 1))
    y_ref = torch.empty_like(xt)
    m.moe_q4_ffn_forward_debug(L, xt, y_ref, ws, path=m.PATH_DECODE)
    torch.cuda.synchronize()
    assert int(m.workspace_views(L, 1, ws)["status"][0].item()) == 0

    y = torch.empty_like(xt)
    t0 = time.time()
    m.moe_q4_ffn_forward_debug(L, xt, y, ws, path=m.PATH_DECODE, force_spin_timeout=True)
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    status = int(m.workspace_views(L, 1, ws)["status"][0].item())
    assert status & m.STATUS_SPIN_TIMEOUT
    # the partial sums are added into y in no fixed order: equal to rounding
    assert rule13(y.cpu().numpy(), y_ref.cpu().numpy(), ORDER_REL)[0]
    assert elapsed < 60.0

    y2 = torch.empty_like(xt)
    m.moe_q4_ffn_forward_debug(L, xt, y2, ws, path=m.PATH_DECODE)
    torch.cuda.synchronize()
    assert int(m.workspace_views(L, 1, ws)["status"][0].item()) == 0
    assert rule13(y2.cpu().numpy(), y_ref.cpu().numpy(), ORDER_REL)[0]
