"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bit-exact: Q8_0 activations, per-block W4A8 integer dot products, top-k
indices given identical logits, the permutation arrays, the requantised
SwiGLU output given the GPU's own h.  Within 1e-3 relative (per element,
against max(|ref|, row rms)): layer outputs with the oracle fed the GPU's
routing and requantised h.  Sizes: every workload the benchmark and the
design use, at full size on the GPU, checked on all tokens where the oracle
is fast and on sampled tokens where it is not (tokens are independent).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import (check_permutation, check_routing, near_tie_tokens, run_forward, rule13,
                         teacher_forced_check, workload)

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU hosts only with -m gpu
    pytest.skip("needs a CUDA device", allow_module_level=True)

import quantized_moe_q4_b200 as m  # noqa: E402  (loads the CUDA library; fails loudly if missing)

PATHS = [m.PATH_AUTO, m.PATH_GROUPED_DP4A, m.PATH_DECODE, m.PATH_TENSOR_CORE]


# --------------------------------------------------------------- building blocks

@pytest.mark.parametrize("T,H", [(1, 512), (5, 2048), (33, 256), (947, 2048)])
def test_quantize_act_bit_exact(T, H):
    rng = np.random.default_rng(T * 7 + H)
    x = rng.standard_normal((T, H)).astype(np.float32)
    x[0, :32] = 0.0                                       # all-zero block
    x[-1, 32:64] = np.float32(127.0) * np.arange(32, dtype=np.float32) / 31   # exact scale 1.0... ties
    x[-1, 64:96] = np.float32([127, 2.5, -2.5, 0.5, -0.5, 4.5] + [0.0] * 26)  # half-way cases
    q, d = m.moe_q4_quantize_act(torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    rq, rd, _ = oracle.quantize_q8_0(x)
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(d.cpu().numpy().view(np.uint16), rd)


def test_quantize_act_overflow_status():
    x = np.zeros((2, 256), np.float32)
    x[1, 40] = 1e9
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, d = m.moe_q4_quantize_act(torch.from_numpy(x).cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & m.STATUS_SCALE_OVERFLOW
    rq, rd, ov = oracle.quantize_q8_0(x)
    assert ov and np.array_equal(d.cpu().numpy().view(np.uint16), rd) and np.array_equal(q.cpu().numpy(), rq)


def test_block_dots_bit_exact():
    rng = np.random.default_rng(3)
    n = 4096
    blocks = rng.integers(0, 256, size=(n, 18), dtype=np.uint8)
    blocks[:, 0:2] = np.frombuffer(np.float16(0.5).tobytes(), np.uint8)
    qa = rng.integers(-127, 128, size=(n, 32), dtype=np.int8)
    blocks[0, 2:] = 0x00
    qa[0] = 127                                           # -8*127*32
    blocks[1, 2:] = 0xFF
    qa[1] = -127                                          # 7*-127*32
    out = m.moe_q4_block_dots(torch.from_numpy(blocks).cuda(), torch.from_numpy(qa).cuda())
    torch.cuda.synchronize()
    ref = np.array([oracle.block_dot(blocks[i], qa[i]) for i in range(n)], np.int32)
    assert np.array_equal(out.cpu().numpy(), ref)
    assert ref[0] == -8 * 127 * 32 and ref[1] == -7 * 127 * 32


@pytest.mark.parametrize("name,T", [("tiny_t16", None), ("decode_t1", 8), ("prefill_t947", None)])
def test_route_standalone(name, T):
    x, lw = workload(name, T=T)
    L = m.Layer.from_host(lw)
    idx, w, logits = m.moe_q4_route(L, torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    v = dict(logits=logits.cpu().numpy(), topk_idx=idx.cpu().numpy(), topk_w=w.cpu().numpy())
    check_routing(lw, x, v)
    assert np.allclose(v["topk_w"].sum(axis=1, dtype=np.float64), 1.0, atol=1e-6)


@pytest.mark.parametrize("name,T", [("tiny_t16", 129), ("tiny_t16", 300), ("prefill_t947", 129),
                                    ("prefill_t947", 1000), ("zipf_t16384", 2048)])
def test_route_many_tokens_cluster_path(name, T):
    """Above 128 tokens the logits come from the cluster kernel (H split over 4
    CTAs, partials added in rank order): ragged token tiles, fewer experts than
    a tile (E = 16), and the sum order fixed, so two calls agree bit for bit."""
    x, lw = workload(name, T=T)
    L = m.Layer.from_host(lw)
    xd = torch.from_numpy(x).cuda()
    idx, w, logits = m.moe_q4_route(L, xd)
    idx2, w2, logits2 = m.moe_q4_route(L, xd)
    torch.cuda.synchronize()
    v = dict(logits=logits.cpu().numpy(), topk_idx=idx.cpu().numpy(), topk_w=w.cpu().numpy())
    check_routing(lw, x, v)
    assert np.array_equal(v["logits"], logits2.cpu().numpy())
    assert np.array_equal(v["topk_idx"], idx2.cpu().numpy())


# --------------------------------------------------------------- whole layer

@pytest.mark.parametrize("path", PATHS)
def test_tiny_full_parity(path):
    x, lw = workload("tiny_t16")
    v = run_forward(lw, x, path=path)
    check_routing(lw, x, v)
    check_permutation(lw, v)
    teacher_forced_check(lw, x, v, np.arange(x.shape[0]))
    assert v["status"][0] == 0
    # free-running against the independent oracle
    ties = near_tie_tokens(lw, x, v)
    assert all(ok for _, ok in ties), f"routing differs beyond near-ties: {ties}"
    same = np.setdiff1d(np.arange(x.shape[0]), [t for t, _ in ties])
    y_free = oracle.moe_forward(lw, x[same])
    ok, worst = rule13(v["y"][same], y_free, 1e-2)
    assert ok, worst


@pytest.mark.parametrize("path", PATHS)
def test_decode_single_token_calls(path):
    x, lw = workload("decode_t1", T=1000)
    for t in (0, 1, 2, 997):
        v = run_forward(lw, x[t:t + 1], path=path)
        check_routing(lw, x[t:t + 1], v)
        check_permutation(lw, v)
        teacher_forced_check(lw, x[t:t + 1], v, [0])


@pytest.mark.parametrize("path", PATHS)
def test_prefill_947_full_size_sampled(path):
    x, lw = workload("prefill_t947")
    v = run_forward(lw, x, path=path)
    check_routing(lw, x, v)
    check_permutation(lw, v)
    rng = np.random.default_rng(0)
    tokens = np.concatenate([[0, 1, 946], rng.choice(947, 29, replace=False)])
    teacher_forced_check(lw, x, v, np.unique(tokens))
    assert v["status"][0] == 0


@pytest.mark.parametrize("path", PATHS)
def test_zipf_16384_full_size_sampled(path):
    x, lw = workload("zipf_t16384")
    v = run_forward(lw, x, path=path, want_h=False)
    check_permutation(lw, v)
    cnt = v["cnt"][:lw.n_experts]
    assert cnt[0] > 2000 and cnt.max() > 20 * max(1, int(np.median(cnt)))     # the skew is there
    rng = np.random.default_rng(1)
    tokens = np.unique(np.concatenate([[0, 16383], rng.choice(16384, 22, replace=False)]))
    teacher_forced_check(lw, x, v, tokens)
    # logits on the sampled tokens
    ref = oracle.router_logits(x[tokens], lw.w_router, lw.router_bias)
    assert np.abs(v["logits"][tokens] - ref).max() <= 2e-5 * np.abs(ref).max()


# --------------------------------------------------------------- edges

@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("T,H,F,E,k,shared", [
    (1, 256, 256, 1, 1, False),       # one dense W4A8 FFN
    (9, 256, 256, 4, 4, True),        # k = E, ragged token tile
    (3, 512, 768, 5, 2, True),        # F = 3*256
    (40, 768, 256, 256, 16, False),   # E = 256, k = 16
    (1, 768, 768, 5, 2, True),        # decode path: odd H and F
    (1, 4096, 512, 16, 4, True),      # decode path: wide H
    (1, 512, 1024, 8, 8, True),       # decode path: more gate/up items than CTAs
    (1, 2048, 2048, 64, 8, True),     # too large for the decode path: falls back
    (1, 256, 512, 256, 16, False),    # decode path: E = 256, k = 16
    (17, 4096, 256, 8, 2, True),      # wide H
])
def test_shapes_and_degenerate_cases(path, T, H, F, E, k, shared):
    x, lw = synth.random_layer(seed=T + H + F + E, H=H, F=F, E=E, k=k, shared=shared, T=T)
    v = run_forward(lw, x, path=path)
    check_routing(lw, x, v)
    check_permutation(lw, v)
    teacher_forced_check(lw, x, v, np.arange(T))


def test_kernel_shared_memory_sizes_in_any_order():
    # the same kernels at a large, a small and again the large shared-memory
    # size: the per-kernel dynamic shared-memory limit must cover all of them
    cases = [(1, 4096, 512, 16, 4, True), (1, 256, 256, 4, 2, True), (1, 4096, 512, 16, 4, True),
             (9, 4096, 256, 8, 2, True), (9, 256, 256, 4, 2, True), (9, 4096, 256, 8, 2, True)]
    for T, H, F, E, k, shared in cases:
        x, lw = synth.random_layer(seed=H + T, H=H, F=F, E=E, k=k, shared=shared, T=T)
        v = run_forward(lw, x)
        teacher_forced_check(lw, x, v, np.arange(T))


def test_zero_tokens_is_a_noop():
    x, lw = workload("tiny_t16")
    L = m.Layer.from_host(lw)
    xe = torch.empty((0, lw.hidden), device="cuda")
    y = m.moe_q4_ffn_forward(L, xe, workspace=m.alloc_workspace(256))
    assert y.shape == (0, lw.hidden)


def test_all_zero_weights_give_zero():
    x, lw = synth.random_layer(seed=4, H=256, F=256, E=4, k=2, shared=True, T=11)
    for a in (lw.w_gate, lw.w_up, lw.w_down, lw.sh_gate, lw.sh_up, lw.sh_down):
        a[..., 2:] = 0x88
    v = run_forward(lw, x)
    assert np.all(v["y"] == 0.0)


def test_forward_host_matches_device():
    x, lw = workload("tiny_t16")
    L = m.Layer.from_host(lw)
    y_dev = m.moe_q4_ffn_forward(L, torch.from_numpy(x).cuda()).cpu().numpy()
    xh = torch.from_numpy(x).pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    ws = m.alloc_workspace(m.moe_q4_ffn_host_workspace_bytes(L, x.shape[0]))
    m.moe_q4_ffn_forward_host(L, xh, yh, ws)
    torch.cuda.synchronize()
    ok, worst = rule13(yh.numpy(), y_dev, 1e-5)
    assert ok, worst


def test_scale_overflow_reported_in_status():
    x, lw = synth.random_layer(seed=8, H=256, F=256, E=4, k=2, shared=False, T=2)
    x[1, 5] = 1e10
    v = run_forward(lw, x, want_h=False)
    assert v["status"][0] & m.STATUS_SCALE_OVERFLOW


@pytest.mark.parametrize("path", [m.PATH_GROUPED_DP4A, m.PATH_TENSOR_CORE])
def test_workspace_reuse_across_sizes(path):
    # one workspace sized for the largest T serves smaller calls; both calls
    # take the same kernel family (different families may round g or u
    # differently in the last bit, which can flip a Q8_0 code of h)
    x, lw = workload("prefill_t947")
    L = m.Layer.from_host(lw)
    ws = m.alloc_workspace(m.moe_q4_ffn_workspace_bytes(L, 947))
    xd = torch.from_numpy(x).cuda()
    y_full = torch.empty_like(xd)
    m.moe_q4_ffn_forward_debug(L, xd, y_full, ws, path=path)
    y_part = torch.empty_like(xd[:100])
    m.moe_q4_ffn_forward_debug(L, xd[:100].contiguous(), y_part, ws, path=path)
    torch.cuda.synchronize()
    ok, worst = rule13(y_part.cpu().numpy(), y_full[:100].cpu().numpy(), 1e-5)
    assert ok, worst
