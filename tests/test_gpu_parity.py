"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bit-exact: Q8_0 activations, per-block W4A8 integer dot products, top-k
indices given identical logits, the permutation arrays, the requantised
SwiGLU output given the GPU's own h.  Within 1e-3 relative (per element,
against max(|ref|, row rms)): layer outputs with the oracle fed the GPU's
routing and requantised h.  Sizes: every workload the benchmark and the
design use, at full size on the GPU, checked on all tokens where the oracle
is fast and on sampled tokens where it is not (tokens are independent).
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import (ORDER_REL, check_permutation, check_routing, expected_block_dots, free_running_report, rule13,
                         run_forward, tile_boundary_tokens, teacher_forced_check, workload)

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU hosts only with -m gpu
    pytest.skip("needs a CUDA device", allow_module_level=True)

import quantized_moe_q4_b200 as m  # noqa: E402  (loads the CUDA library; fails loudly if missing)

# every kernel family: automatic choice, streaming dp4a, fused decode (T = 1;
# other T take the grouped paths), tensor cores with 32-, 64- and 128-slot tiles
PATHS = [m.PATH_AUTO, m.PATH_GROUPED_DP4A, m.PATH_DECODE, m.PATH_TENSOR_CORE_N32, m.PATH_TENSOR_CORE_N64,
         m.PATH_TENSOR_CORE_N128]


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

def check_free_running(name, path, lw, x, v, tokens):
    """The free-running report against the independent oracle (printed):
    routing may differ only at near-ties; a token with identical routing and
    identical requantised SwiGLU output is within 1e-3 norm-wise (in practice
    binary32 rounding); a requantised code moves by at most one step, which
    moves its token by less than 1e-2 norm-wise; and at least 99% of the
    tokens with identical routing are within 1e-3."""
    rep = free_running_report(lw, x, v, tokens)
    print(f"free-running {name} path {path}: {rep}")
    assert rep["other"] == 0, rep
    assert rep["row_err"] <= 1e-3, rep
    assert rep["big_flips"] == 0, rep
    assert rep["requant_row_err"] <= 1e-2, rep
    assert rep["within_1e3"] >= 0.99, rep
    return rep


@pytest.mark.parametrize("path", PATHS)
def test_tiny_full_parity(path):
    x, lw = workload("tiny_t16")
    v = run_forward(lw, x, path=path)
    check_routing(lw, x, v)
    check_permutation(lw, v)
    teacher_forced_check(lw, x, v, np.arange(x.shape[0]))
    assert v["status"][0] == 0
    check_free_running("tiny_t16", path, lw, x, v, np.arange(x.shape[0]))


@pytest.mark.parametrize("path", PATHS)
def test_decode_single_token_calls(path):
    x, lw = workload("decode_t1", T=1000)
    for t in (0, 1, 2, 997):
        v = run_forward(lw, x[t:t + 1], path=path)
        check_routing(lw, x[t:t + 1], v)
        check_permutation(lw, v)
        teacher_forced_check(lw, x[t:t + 1], v, [0])


@pytest.mark.parametrize("path", PATHS)
def test_prefill_947_every_token(path):
    """All 947 tokens teacher-forced and free-running."""
    x, lw = workload("prefill_t947")
    v = run_forward(lw, x, path=path)
    check_routing(lw, x, v)
    check_permutation(lw, v)
    teacher_forced_check(lw, x, v, np.arange(947))
    assert v["status"][0] == 0
    check_free_running("prefill_t947", path, lw, x, v, np.arange(947))


@pytest.mark.parametrize("path", PATHS)
def test_zipf_16384_tile_boundaries(path):
    """Full size on the device; the oracle checks the first and last slot of
    every 64-slot tile (the tensor-core tile; every eighth 8-slot tile of the
    streaming path) of the ten most loaded experts and of the shared expert,
    the first and last tokens, and a random sample; free-running on the same
    tokens."""
    x, lw = workload("zipf_t16384")
    v = run_forward(lw, x, path=path, want_h=False)
    check_permutation(lw, v)
    T, E = x.shape[0], lw.n_experts
    cnt = v["cnt"][:E]
    assert cnt[0] > 2000 and cnt.max() > 20 * max(1, int(np.median(cnt)))     # the skew is there
    heavy = np.argsort(-cnt, kind="stable")[:10]
    rng = np.random.default_rng(1)
    tokens = np.unique(np.concatenate([tile_boundary_tokens(lw, T, v, list(heavy) + [E], 64),
                                       [0, T - 1], rng.choice(T, 256, replace=False)]))
    teacher_forced_check(lw, x, v, tokens)
    # logits on the checked tokens
    ref = oracle.router_logits(x[tokens], lw.w_router, lw.router_bias)
    assert np.abs(v["logits"][tokens] - ref).max() <= 2e-5 * np.abs(ref).max()
    check_free_running("zipf_t16384", path, lw, x, v, tokens)


# --------------------------------------------------------------- per-block integer sums

def _capture(lw, x, path, down, g, rb, R):
    import quantized_moe_q4_b200 as mm
    from gpu_helpers import device_layer
    L = device_layer(lw)
    xd = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    T = x.shape[0]
    ws = mm.alloc_workspace(mm.moe_q4_ffn_workspace_bytes(L, T))
    off = mm.workspace_views(L, T, ws)
    y = torch.empty_like(xd)
    # a first call fills the permutation, which sizes the capture buffer
    mm.moe_q4_ffn_forward_debug(L, xd, y, ws, path=path)
    torch.cuda.synchronize()
    c = int(off["off"][g + 1].item() - off["off"][g].item())
    K = lw.ffn if down else lw.hidden
    out = torch.full((c, R, K // 32), -(2 ** 31), dtype=torch.int32, device="cuda")
    mm.moe_q4_ffn_forward_debug(L, xd, y, ws, path=path, block_dots=(out, down, g, rb))
    torch.cuda.synchronize()
    v = {k: t.cpu().numpy() for k, t in mm.workspace_views(L, T, ws).items()}
    return out.cpu().numpy(), v


def _groups_to_capture(v, E, tile):
    """A routed group whose last tile is ragged, the routed group with the
    most slots (several tiles), and the shared expert."""
    cnt = v["cnt"][:E]
    ragged = [g for g in range(E) if cnt[g] > 0 and cnt[g] % tile]
    return sorted({ragged[0], int(np.argmax(cnt)), E})


@pytest.mark.parametrize("path,R,tile", [(m.PATH_TENSOR_CORE_N32, 128, 32), (m.PATH_TENSOR_CORE_N64, 128, 64),
                                         (m.PATH_TENSOR_CORE_N128, 128, 128), (m.PATH_GROUPED_DP4A, 64, 8)])
@pytest.mark.parametrize("down", [False, True])
def test_block_dots_of_the_projection_kernels_bit_exact(path, R, tile, down):
    """The per-block integer sums I_b inside the grouped projection kernels
    (the tensor-core path: the MMA accumulator of one block before the
    rescale), captured for whole row blocks of several expert groups of the
    947-token prefill, equal the oracle's block dot products bit for bit."""
    x, lw = workload("prefill_t947")
    T, E = x.shape[0], lw.n_experts
    _, v0 = _capture(lw, x, path, down, E, 0, R)
    n_rb = (lw.hidden if down else 2 * lw.ffn) // R
    for g in _groups_to_capture(v0, E, tile):
        if g == E and not down:
            continue   # 947 slots x all of H: covered at a smaller size by the extremes test
        for rb in sorted({0, n_rb - 1, (g * 7) % n_rb}):
            got, v = _capture(lw, x, path, down, g, rb, R)
            assert np.array_equal(v["hq"], v0["hq"]) and np.array_equal(v["off"], v0["off"])
            ref = expected_block_dots(lw, T, v, down, g, rb, R)
            assert got.shape == ref.shape
            bad = np.argwhere(got != ref)
            assert bad.size == 0, f"group {g} row block {rb}: {len(bad)} block sums differ, first {bad[:3]}"


@pytest.mark.parametrize("path,R", [(m.PATH_TENSOR_CORE_N32, 128), (m.PATH_TENSOR_CORE_N64, 128),
                                    (m.PATH_TENSOR_CORE_N128, 128), (m.PATH_GROUPED_DP4A, 64)])
def test_block_dots_extreme_values(path, R):
    """All nibbles 0 or 15 against activations at +-127 (Q8_0 of rows whose
    blocks hold one large value of either sign and equal smaller ones): the
    extremes of I_b, |I_b| up to 8 * 127 * 32, stay exact."""
    x, lw = synth.random_layer(seed=12, H=512, F=256, E=4, k=2, shared=True, T=150)
    lw.w_gate[..., 2:] = 0x00
    lw.w_up[..., 2:] = 0xFF
    lw.sh_gate[..., 2:10] = 0x00
    lw.sh_gate[..., 10:] = 0xFF
    x[:, :] = 1.0
    x[1::2] = -1.0                  # every code +127 in even rows, -127 in odd rows
    T, E = x.shape[0], lw.n_experts
    for g in range(E + 1):
        got, v = _capture(lw, x, path, False, g, 0, R)
        ref = expected_block_dots(lw, T, v, False, g, 0, R)
        assert np.array_equal(got, ref), g
        if g < E and got.size:
            assert np.abs(got).max() == 8 * 127 * 32


# --------------------------------------------------------------- edges

@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("T,H,F,E,k,shared", [
    (1, 256, 256, 1, 1, False),       # one dense W4A8 FFN
    (9, 256, 256, 4, 4, True),        # k = E, ragged token tile
    (3, 512, 768, 5, 2, True),        # F = 3*256
    (40, 768, 256, 256, 16, False),   # E = 256, k = 16
    (1, 768, 768, 5, 2, True),        # decode path: odd H and F
    (1, 4096, 512, 16, 4, True),      # H above the decode path's 2560: falls back
    (1, 2560, 512, 16, 4, True),      # decode path: the widest H
    (1, 512, 1024, 8, 8, True),       # 288 h blocks, more than one wave: falls back
    (1, 2048, 2048, 64, 8, True),     # too large for the decode path: falls back
    (1, 256, 256, 256, 16, False),    # decode path: E = 256 (8 logits a lane in the top-k), k = 16
    (1, 512, 256, 200, 8, True),      # decode path: E = 200, not a multiple of 32
    (17, 4096, 256, 8, 2, True),      # wide H
    (5, 1536, 1792, 12, 3, True),     # rows of 48 and 56 blocks (streaming chunks of 24 and 8)
    (3, 2304, 2560, 6, 2, False),     # rows of 72 and 80 blocks (chunks of 24 and 16)
])
def test_shapes_and_degenerate_cases(path, T, H, F, E, k, shared):
    x, lw = synth.random_layer(seed=T + H + F + E, H=H, F=F, E=E, k=k, shared=shared, T=T)
    v = run_forward(lw, x, path=path)
    check_routing(lw, x, v)
    check_permutation(lw, v)
    teacher_forced_check(lw, x, v, np.arange(T))


@pytest.mark.parametrize("path", PATHS)
def test_routing_with_exact_ties(path):
    """Ten experts with identical router rows get identical logits on every
    path (the same products summed in the same order), at the top of the
    ranking: with k = 8 the top-k takes the eight lowest of their indices, in
    index order, exactly as the oracle's top-k of the device's own logits."""
    T = 1 if path == m.PATH_DECODE else 24
    x, lw = synth.random_layer(seed=99, H=256, F=256, E=64, k=8, shared=True, T=T)
    tied = [1, 3, 7, 12, 20, 30, 41, 50, 55, 63]
    row = lw.w_router[41].copy()
    if float(np.dot(x[0].astype(np.float64), row)) < 0:
        row = -row                                   # token 0 ranks the tied experts first
    Wr = lw.w_router.copy()
    for e in tied:
        Wr[e] = 10 * row
    lw = dataclasses.replace(lw, w_router=Wr)
    v = run_forward(lw, x, path=path, L=m.Layer.from_host(lw))
    check_routing(lw, x, v)
    check_permutation(lw, v)
    assert v["topk_idx"][0].tolist() == tied[:8]
    teacher_forced_check(lw, x, v, np.arange(T))


def test_kernel_shared_memory_sizes_in_any_order():
    # the same kernels at a large, a small and again the large shared-memory
    # size: the per-kernel dynamic shared-memory limit must cover all of them
    cases = [(1, 2560, 512, 16, 4, True), (1, 256, 256, 4, 2, True), (1, 2560, 512, 16, 4, True),
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


@pytest.mark.parametrize("pinned", [True, False])
def test_forward_host_single_token(pinned):
    """One token through the host entry: with page-locked x and y the decode
    kernels read x and write y over the bus (no copy node); with pageable
    memory the entry falls back to stream copies.  Either way the result is
    the device forward's, call after call."""
    x, lw = workload("decode_t1", T=1000)
    L = m.Layer.from_host(lw)
    ws = m.alloc_workspace(m.moe_q4_ffn_host_workspace_bytes(L, 1))
    for t in (0, 5, 999):
        xt = torch.from_numpy(x[t:t + 1].copy())
        y_dev = m.moe_q4_ffn_forward(L, xt.cuda()).cpu().numpy()
        xh = xt.pin_memory() if pinned else xt
        yh = torch.full_like(xh, float("nan"))
        yh = yh.pin_memory() if pinned else yh
        m.moe_q4_ffn_forward_host(L, xh, yh, ws)
        torch.cuda.synchronize()
        ok, worst = rule13(yh.numpy(), y_dev, ORDER_REL)
        assert ok, worst


def test_forward_host_back_to_back():
    """One-token host calls enqueued with no synchronisation between them: a
    call whose x is the previous call's y (the entry must not read it before
    that y has landed), then calls on distinct buffers (x read early, while
    the previous call finishes).  Each output must be the device forward of
    the input it was given; outputs start as NaN so a stale read shows."""
    x, lw = workload("decode_t1", T=1000)
    L = m.Layer.from_host(lw)
    ws = m.alloc_workspace(m.moe_q4_ffn_host_workspace_bytes(L, 1))
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).pin_memory()
    nan = lambda: torch.full((1, lw.hidden), float("nan")).pin_memory()
    x0, x1, x2 = pin(x[0:1]), pin(x[1:2]), pin(x[2:3])
    ya, yb, yc, yd, ye = nan(), nan(), nan(), nan(), nan()
    m.moe_q4_ffn_forward_host(L, x0, ya, ws)
    m.moe_q4_ffn_forward_host(L, ya, yb, ws)        # x = the previous call's y
    m.moe_q4_ffn_forward_host(L, x1, yc, ws)        # distinct buffers from here on
    m.moe_q4_ffn_forward_host(L, x2, yd, ws)
    m.moe_q4_ffn_forward_host(L, yd, ye, ws)        # aliasing again
    torch.cuda.synchronize()
    for xin, yout in ((x0, ya), (ya, yb), (x1, yc), (x2, yd), (yd, ye)):
        assert np.all(np.isfinite(yout.numpy()))
        y_dev = m.moe_q4_ffn_forward(L, xin.cuda()).cpu().numpy()
        ok, worst = rule13(yout.numpy(), y_dev, ORDER_REL)
        assert ok, worst


def test_decode_kernel_timer():
    """The fused T = 1 path's device timer: one count per call, the span from
    the dependency wait no longer than the span from the kernel's start, both
    positive and below a millisecond a call; results unchanged by timing."""
    x, lw = workload("decode_t1", T=8)
    L = m.Layer.from_host(lw)
    ws = m.alloc_workspace(m.moe_q4_ffn_workspace_bytes(L, 1))
    timer = torch.zeros(3, dtype=torch.int64, device="cuda")
    xd = torch.from_numpy(x).cuda()
    y_t, y_u = torch.empty_like(xd), torch.empty_like(xd)
    for t in range(8):
        m.moe_q4_ffn_forward_debug(L, xd[t:t + 1], y_t[t:t + 1], ws, path=m.PATH_DECODE, decode_kernel_ns=timer)
        m.moe_q4_ffn_forward_debug(L, xd[t:t + 1], y_u[t:t + 1], ws, path=m.PATH_DECODE)
    torch.cuda.synchronize()
    ready_ns, n, resident_ns = timer.cpu().tolist()
    assert n == 8
    assert 0 < ready_ns <= resident_ns < 8 * 1_000_000
    ok, worst = rule13(y_t.cpu().numpy(), y_u.cpu().numpy(), ORDER_REL)
    assert ok, worst


def test_scale_overflow_reported_in_status():
    x, lw = synth.random_layer(seed=8, H=256, F=256, E=4, k=2, shared=False, T=2)
    x[1, 5] = 1e10
    v = run_forward(lw, x, want_h=False)
    assert v["status"][0] & m.STATUS_SCALE_OVERFLOW


@pytest.mark.parametrize("path", [m.PATH_GROUPED_DP4A, m.PATH_TENSOR_CORE_N32, m.PATH_TENSOR_CORE_N64,
                                  m.PATH_TENSOR_CORE_N128])
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
