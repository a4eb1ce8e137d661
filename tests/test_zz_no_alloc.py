"""moe_q4_ffn_forward_noalloc: the layer for callers that cannot allocate
device memory (their memory is reserved up front by a host runtime, they may
not pay for cudaMalloc's implicit synchronisation mid-step, or they record CUDA
graphs).  It uses the library's static device scratch instead of a caller
workspace; its results must match moe_q4_ffn_forward's, call after call.

Collected last on purpose (file name), so a run that stops at the first
failure has run every other test before this one.
"""
import numpy as np
import pytest
import torch

import synth
from gpu_helpers import rule13

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import quantized_moe_q4_b200 as m  # noqa: E402


def _reference(L, x):
    """The existing entry point with a caller-allocated workspace."""
    ws = m.alloc_workspace(m.moe_q4_ffn_workspace_bytes(L, x.shape[0]))
    y = m.moe_q4_ffn_forward(L, x, workspace=ws)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def test_noalloc_matches_forward_on_two_calls_in_a_row():
    x1, lw1 = synth.workload_inputs("tiny_t16", seed=0)
    x2, lw2 = synth.workload_inputs("decode_t1", seed=0, T=300)
    L1, L2 = m.Layer.from_host(lw1), m.Layer.from_host(lw2)
    xd1, xd2 = torch.from_numpy(x1).cuda(), torch.from_numpy(x2[1:2].copy()).cuda()
    xd3 = torch.from_numpy(x2[:256].copy()).cuda()
    ref1, ref2, ref3 = _reference(L1, xd1), _reference(L2, xd2), _reference(L2, xd3)
    # calls in a row on the shared scratch: a 16-token layer (streaming
    # kernels), a one-token call of a different layer (fused decode kernels),
    # then 256 tokens of that layer (tensor-core kernels, another layout of
    # the same array)
    y1 = m.moe_q4_ffn_forward_noalloc(L1, xd1)
    y2 = m.moe_q4_ffn_forward_noalloc(L2, xd2)
    y3 = m.moe_q4_ffn_forward_noalloc(L2, xd3)
    torch.cuda.synchronize()
    for y, ref in ((y1, ref1), (y2, ref2), (y3, ref3)):
        ok, worst = rule13(y.cpu().numpy(), ref, 1e-3)
        assert ok, f"no-alloc output differs from moe_q4_ffn_forward: worst {worst:.3e}"
    # and once more with the first layer, after the scratch held the second call
    y3 = m.moe_q4_ffn_forward_noalloc(L1, xd1)
    torch.cuda.synchronize()
    ok, worst = rule13(y3.cpu().numpy(), ref1, 1e-3)
    assert ok, worst


def test_noalloc_rejects_problems_beyond_the_scratch():
    _, lw = synth.workload_inputs("decode_t1", seed=0, T=1)
    L = m.Layer.from_host(lw)
    limit = m.moe_q4_ffn_workspace_bytes(L, 542)
    assert limit <= (4 << 20) < m.moe_q4_ffn_workspace_bytes(L, 543)
    x = torch.zeros((543, lw.hidden), device="cuda")
    y = torch.full_like(x, 7.0)
    with pytest.raises(m.MoeQ4Error) as e:
        m.moe_q4_ffn_forward_noalloc(L, x, y)
    assert e.value.code == -4
    torch.cuda.synchronize()
    assert bool(torch.all(y == 7.0))          # nothing was enqueued
