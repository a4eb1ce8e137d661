"""Host-streamed experts: the expert matrices in page-locked host memory,
the routing-selected experts copied to the device per call.  Results equal
the resident layer's (within the order of the binary32 partial sums added
into y), exactly the selected experts are staged, and pageable host memory
is refused before anything runs."""
import numpy as np
import pytest
import torch

from gpu_helpers import ORDER_REL, check_permutation, check_routing, rule13, teacher_forced_check, workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import quantized_moe_q4_b200 as m  # noqa: E402


def _both(name, T=None):
    x, lw = workload(name, T=T)
    return x, lw, m.Layer.from_host(lw), m.Layer.from_host_pinned(lw)


def test_streamed_decode_tokens_match_resident():
    x, lw, Ld, Lh = _both("decode_t1", T=1000)
    for t in (0, 1, 2, 999):
        xt = torch.from_numpy(x[t:t + 1].copy()).cuda()
        y_res = m.moe_q4_ffn_forward(Ld, xt)
        y_str = m.moe_q4_ffn_forward_streamed(Lh, xt)
        torch.cuda.synchronize()
        ok, worst = rule13(y_str.cpu().numpy(), y_res.cpu().numpy(), ORDER_REL)
        assert ok, worst


@pytest.mark.parametrize("name,T", [("prefill_t947", 16), ("prefill_t947", None), ("tiny_t16", None)])
def test_streamed_matches_resident(name, T):
    x, lw, Ld, Lh = _both(name)
    x = x if T is None else x[:T]
    xd = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    y_res = m.moe_q4_ffn_forward(Ld, xd).cpu().numpy()
    y_str = m.moe_q4_ffn_forward_streamed(Lh, xd).cpu().numpy()
    ok, worst = rule13(y_str, y_res, 1e-5)
    assert ok, worst


@pytest.mark.parametrize("name,T", [("decode_t1", 1), ("prefill_t947", 16), ("prefill_t947", None)])
def test_streamed_against_the_oracle(name, T):
    """The streamed layer teacher-forced against the oracle on every token:
    its own routing (bit-exact given its logits), permutation, requantised
    SwiGLU output (the oracle's Q8_0 of the device's h) and output."""
    x, lw = workload(name, T=1000 if name == "decode_t1" else None)
    x = np.ascontiguousarray(x if T is None else x[:T])
    T = x.shape[0]
    Lh = m.Layer.from_host_pinned(lw)
    xd = torch.from_numpy(x).cuda()
    y = torch.empty_like(xd)
    ws = m.alloc_workspace(m.moe_q4_ffn_workspace_bytes(Lh, T))
    m.moe_q4_ffn_forward_streamed(Lh, xd, y, workspace=ws)
    torch.cuda.synchronize()
    v = {k: t.cpu().numpy() for k, t in m.workspace_views(Lh, T, ws).items()}
    v["y"] = y.cpu().numpy()
    check_routing(lw, x, v)
    check_permutation(lw, v)
    teacher_forced_check(lw, x, v, np.arange(T))
    assert v["status"][0] == 0


def test_only_selected_experts_are_staged():
    x, lw, Ld, Lh = _both("decode_t1", T=1000)
    xt = torch.from_numpy(x[:3].copy()).cuda()
    staging = m.alloc_workspace(m.moe_q4_staging_bytes(Lh))
    staging.fill_(0xA5)
    ws = m.alloc_workspace(m.moe_q4_ffn_workspace_bytes(Lh, 3))
    m.moe_q4_ffn_forward_streamed(Lh, xt, workspace=ws, staging=staging)
    torch.cuda.synchronize()
    idx = m.workspace_views(Lh, 3, ws)["topk_idx"].cpu().numpy()
    active = set(idx.ravel().tolist())
    st = staging.cpu().numpy()
    E, F, H = lw.n_experts, lw.ffn, lw.hidden
    gu = F * (H // 32) * 18
    for e in range(E):
        seg = st[e * gu:(e + 1) * gu]
        if e in active:
            assert np.array_equal(seg, lw.w_gate[e].reshape(-1))
        else:
            assert np.all(seg == 0xA5), f"expert {e} was staged without being selected"


def test_pageable_host_memory_is_refused():
    x, lw = workload("tiny_t16")
    d = lambda a: None if a is None else torch.from_numpy(a).cuda()  # noqa: E731
    h = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a))  # noqa: E731  (not pinned)
    L = m.Layer(lw.hidden, lw.ffn, lw.n_experts, lw.top_k, d(lw.w_router), d(lw.router_bias),
                h(lw.w_gate), h(lw.w_up), h(lw.w_down))
    with pytest.raises(m.MoeQ4Error) as e:
        m.moe_q4_ffn_forward_streamed(L, torch.from_numpy(x).cuda())
    assert e.value.code == -1
