"""The device status word and non-finite inputs, on the GPU.

Routing: a NaN router logit ranks below every number (equal keys go to the
lower expert index), so the top-k of every token is k distinct experts in
[0, E) whatever the logits hold, and the NONFINITE_LOGIT bit reports it.
These are first checked through moe_q4_route alone, which never uses the
indices to address memory, and only then through whole forwards.

Stack: moe_q4_stack_forward clears the status word once and every layer ORs
its conditions into it, so a binary16 overflow in layer 2 of 4 is still
reported after the call.
"""
import numpy as np
import pytest
import torch

import synth
from gpu_helpers import check_permutation, run_forward, teacher_forced_check

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import quantized_moe_q4_b200 as m  # noqa: E402


def expected_topk(logits, k):
    """k experts per token: NaN as -inf, descending, equal keys by index."""
    key = np.where(np.isnan(logits), -np.inf, logits).astype(np.float64)
    E = logits.shape[1]
    order = np.lexsort((np.broadcast_to(np.arange(E), key.shape), -key), axis=-1)
    return order[:, :k].astype(np.int32)


def _bias(E, nan=(), neg_inf=(), pos_inf=()):
    b = np.zeros(E, np.float32)
    b[list(nan)] = np.nan
    b[list(neg_inf)] = -np.inf
    b[list(pos_inf)] = np.inf
    return b


@pytest.mark.parametrize("T", [1, 16, 300])
@pytest.mark.parametrize("case", ["some", "all_nan", "most_nonfinite"])
def test_route_with_nonfinite_logits_keeps_indices_in_range(T, case):
    x, lw = synth.random_layer(seed=5, H=512, F=256, E=16, k=4, shared=False, T=T)
    if case == "some":
        lw.router_bias = _bias(16, nan=(0, 3), neg_inf=(5,), pos_inf=(9,))
    elif case == "all_nan":
        lw.router_bias = np.full(16, np.nan, np.float32)
    else:   # fewer finite experts than k: the rest are filled by index
        lw.router_bias = _bias(16, nan=range(2, 16))
        lw.router_bias[1] = -np.inf
    L = m.Layer.from_host(lw)
    idx, w, logits = m.moe_q4_route(L, torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    idx, lg = idx.cpu().numpy(), logits.cpu().numpy()
    assert idx.min() >= 0 and idx.max() < 16
    for t in range(T):
        assert len(set(idx[t])) == 4, idx[t]
    assert np.array_equal(idx, expected_topk(lg, 4))
    if case == "all_nan":
        assert np.all(idx == np.arange(4))


@pytest.mark.parametrize("path,T", [(m.PATH_DECODE, 1), (m.PATH_GROUPED_DP4A, 16), (m.PATH_TENSOR_CORE, 200),
                                    (m.PATH_AUTO, 1), (m.PATH_AUTO, 16)])
def test_forward_with_a_nan_expert_bias(path, T):
    """Experts whose bias is NaN or -inf are never chosen while k finite ones
    remain; the layer is otherwise exact and the status word says so."""
    x, lw = synth.random_layer(seed=6, H=512, F=256, E=16, k=4, shared=True, T=T)
    lw.router_bias = _bias(16, nan=(2, 11), neg_inf=(7,))
    v = run_forward(lw, x, path=path)
    assert v["status"][0] & m.STATUS_NONFINITE_LOGIT
    assert not v["status"][0] & m.STATUS_BAD_EXPERT_INDEX
    idx = v["topk_idx"]
    assert idx.min() >= 0 and idx.max() < 16 and not np.isin(idx, [2, 7, 11]).any()
    assert np.array_equal(idx, expected_topk(v["logits"], 4))
    check_permutation(lw, v)
    teacher_forced_check(lw, x, v, np.arange(T))
    assert np.all(np.isfinite(v["y"]))


@pytest.mark.parametrize("path,T", [(m.PATH_DECODE, 1), (m.PATH_GROUPED_DP4A, 16), (m.PATH_TENSOR_CORE, 200)])
def test_forward_with_all_logits_nan_stays_in_bounds(path, T):
    x, lw = synth.random_layer(seed=7, H=512, F=256, E=16, k=4, shared=True, T=T)
    lw.router_bias = np.full(16, np.nan, np.float32)
    v = run_forward(lw, x, path=path, want_h=False)
    assert v["status"][0] & m.STATUS_NONFINITE_LOGIT
    assert np.all(v["topk_idx"] == np.arange(4))
    check_permutation(lw, v)


def _overflow_layer(lw):
    """Gate and up scales of 1000: SwiGLU outputs near 1e10, beyond the
    binary16 Q8_0 scale range (block amax / 127 > 65504)."""
    big = np.frombuffer(np.float16(1000.0).tobytes(), np.uint8)
    for a in (lw.w_gate, lw.w_up, lw.sh_gate, lw.sh_up):
        a[..., 0:2] = big
    return lw


@pytest.mark.parametrize("T", [1, 64, 256])
def test_stack_status_accumulates_over_layers(T):
    H, F, E, k = 512, 256, 16, 4
    lws = [synth.stack_layer(l, H, F, E, k, True, seed=3) for l in range(4)]
    _overflow_layer(lws[1])
    layers = [m.Layer.from_host(lw) for lw in lws]
    x0 = torch.from_numpy(synth.stack_inputs(T, H, seed=3)).cuda()
    ws = m.alloc_workspace(m.moe_q4_stack_workspace_bytes(layers[0], T))
    status_off = 2 * (((T * H * 4) + 255) // 256 * 256)

    def status():
        torch.cuda.synchronize()
        return int(ws[status_off:status_off + 4].view(torch.int32).item())

    # the first layer alone is clean; a stale word from an earlier call is cleared
    ws[status_off:status_off + 4].view(torch.int32).fill_(0x7ffffff0)
    x = x0.clone()
    m.moe_q4_stack_forward(layers[:1], x, workspace=ws)
    assert status() == 0
    # layer 2 overflows; layers 3 and 4 then see non-finite activations, and
    # the overflow bit set in layer 2 is still there after the call
    x = x0.clone()
    m.moe_q4_stack_forward(layers, x, workspace=ws)
    st = status()
    assert st & m.STATUS_SCALE_OVERFLOW, hex(st)
    assert not st & m.STATUS_BAD_EXPERT_INDEX
    # the next call starts from a clear word
    x = x0.clone()
    m.moe_q4_stack_forward(layers[:1], x, workspace=ws)
    assert status() == 0
