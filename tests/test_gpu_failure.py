"""Failure detection without a GPU fault: the fused decode kernel's grid
barrier is made to wait for one CTA more than exist (a flag nothing will
set).  Its wait is bounded, so it gives up, the kernel finishes (every CTA
did write its rows), the status word reports the timeout, the results are
still right, and the context stays usable: the next call is clean."""
import time

import pytest
import torch

from gpu_helpers import workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import quantized_moe_q4_b200 as m  # noqa: E402


def test_decode_barrier_timeout_reported_and_recovered():
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
    assert torch.equal(y, y_ref)
    assert elapsed < 60.0

    y2 = torch.empty_like(xt)
    m.moe_q4_ffn_forward_debug(L, xt, y2, ws, path=m.PATH_DECODE)
    torch.cuda.synchronize()
    assert int(m.workspace_views(L, 1, ws)["status"][0].item()) == 0
    assert torch.equal(y2, y_ref)
