"""The 40-layer stack (x <- x + MoE_l(RMSNorm(x)), 2048/512, 128 experts
top-8 + shared, independently seeded layers) on the device against the
oracle: the glue kernel bit for bit (RMSNorm within one binary32 ulp), every
layer teacher-forced on sampled tokens with the GPU's own layer input, the
one-call stack entry against the layer-by-layer composition, and a
free-running oracle run through all 40 layers on a few tokens."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import check_routing, rule13, run_forward, teacher_forced_check, tile_boundary_tokens

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import quantized_moe_q4_b200 as m  # noqa: E402

EPS = 1e-6


def ulps(a, b):
    ia = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    ib = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    ia = np.where(ia < 0, np.int64(-2**31) - ia, ia)
    ib = np.where(ib < 0, np.int64(-2**31) - ib, ib)
    return np.abs(ia - ib)


def test_residual_rmsnorm_matches_oracle():
    rng = np.random.default_rng(11)
    T, H = 37, 2048                                   # ragged: not a multiple of the 4 rows a CTA takes
    x = (rng.standard_normal((T, H)) * 3).astype(np.float32)
    y = rng.standard_normal((T, H)).astype(np.float32)
    x[0] = 0.0
    y[0] = 0.0                                         # all-zero row: rms = sqrt(eps), xn = 0
    x[1] = 1e-30                                       # far below eps
    x[2] *= np.float32(1e25)                           # squares overflow binary32, not binary64
    xd, yd = torch.from_numpy(x).cuda(), torch.from_numpy(y).cuda()
    xn = m.moe_q4_residual_rmsnorm(xd, yd, eps=EPS)
    torch.cuda.synchronize()
    x1 = oracle.residual_add(x, y)
    assert np.array_equal(xd.cpu().numpy(), x1)
    u = ulps(xn.cpu().numpy(), oracle.rmsnorm(x1, EPS))
    assert u.max() <= 1 and np.count_nonzero(u) <= 4
    assert np.all(xn.cpu().numpy()[0] == 0)
    # without y: x unchanged, xn of x
    xd2 = torch.from_numpy(x).cuda()
    xn2 = m.moe_q4_residual_rmsnorm(xd2, None, eps=EPS)
    torch.cuda.synchronize()
    assert np.array_equal(xd2.cpu().numpy(), x)
    assert ulps(xn2.cpu().numpy(), oracle.rmsnorm(x, EPS)).max() <= 1
    # without xn: the residual add alone
    f = m.library().moe_q4_residual_rmsnorm
    assert f(ctypes.c_void_p(xd2.data_ptr()), ctypes.c_void_p(yd.data_ptr()), T, H, EPS, None,
             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    torch.cuda.synchronize()
    assert np.array_equal(xd2.cpu().numpy(), x1)


def _run_stack(T, n_check, seed=0):
    """Layer by layer through the public entries, every layer checked against
    the oracle; returns (x0, the final x, device layers, oracle free run)."""
    c = synth.WORKLOADS["stack40"]
    H, F, E, k, NL = c["H"], c["F"], c["E"], c["k"], c["layers"]
    x0 = synth.stack_inputs(T, H, seed)
    x = torch.from_numpy(x0).cuda()
    rng = np.random.default_rng(T)
    free_tok = np.array([0, T - 1])
    x_free = x0[free_tok].copy()
    layers, y, x_after2 = [], None, None
    for l in range(NL):
        lw = synth.stack_layer(l, H, F, E, k, c["shared"], seed)
        L = m.Layer.from_host(lw)
        layers.append(L)
        xn = m.moe_q4_residual_rmsnorm(x, y, eps=EPS)
        torch.cuda.synchronize()
        x_np, xn_np = x.cpu().numpy(), xn.cpu().numpy()
        if l == 2:
            x_after2 = x_np.copy()
        u = ulps(xn_np, oracle.rmsnorm(x_np, EPS))
        assert u.max() <= 1, f"layer {l}: RMSNorm off by {u.max()} ulp"
        v = run_forward(lw, xn_np, want_h=False, L=L)
        check_routing(lw, xn_np, v)
        # the first and last slot of every 64-slot tile of the layer's most
        # loaded expert and of the shared expert, plus a random sample
        heavy = int(np.argmax(v["cnt"][:E]))
        toks = np.unique(np.concatenate([[0, T - 1], rng.choice(T, n_check, replace=False),
                                         tile_boundary_tokens(lw, T, v, [heavy, E], 64)]))
        teacher_forced_check(lw, xn_np, v, toks)
        assert v["status"][0] == 0, f"layer {l}: status {v['status'][0]}"
        y = torch.from_numpy(v["y"]).cuda()
        x_free = oracle.residual_add(x_free, oracle.moe_forward(lw, oracle.rmsnorm(x_free, EPS)))
        del lw
    m.moe_q4_residual_rmsnorm(x, y, eps=EPS)
    torch.cuda.synchronize()
    return x0, x.cpu().numpy(), layers, (free_tok, x_free), x_after2


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return np.linalg.norm(a - b, axis=-1) / np.linalg.norm(b, axis=-1)


def _check_one_call(x0, x_layerwise, x_after2, layers):
    # two layers through the one-call entry reproduce the layer-by-layer
    # composition: the same kernels, only the order of the fp32 atomic combine
    # differs (a last-bit effect that can flip at most a rare Q8_0 code)
    x = torch.from_numpy(x0).cuda()
    m.moe_q4_stack_forward(layers[:2], x, eps=EPS)
    torch.cuda.synchronize()
    x2 = x.cpu().numpy()
    T = x0.shape[0]
    bad = [t for t in range(T) if not rule13(x2[t:t + 1], x_after2[t:t + 1], 1e-3)[0]]
    # measured: 0 of 64 and 2 of 4096 tokens (a flipped code that moved a
    # second-layer routing near-tie)
    assert len(bad) <= max(1, T // 512), f"tokens off after two layers of the one-call stack: {bad}"
    # all 40 layers: that last-bit difference is amplified by 40 rounds of
    # requantisation and routing; report how far the two runs drift apart
    x = torch.from_numpy(x0).cuda()
    m.moe_q4_stack_forward(layers, x, eps=EPS)
    torch.cuda.synchronize()
    xs = x.cpu().numpy()
    assert np.all(np.isfinite(xs))
    e = rel_l2(xs, x_layerwise)
    print(f"one-call vs layer-by-layer after {len(layers)} layers: relative L2 per token "
          f"median {np.median(e):.2e}, max {e.max():.2e}")
    # most tokens agree to binary32 precision; a few drift once a routing
    # decision on a near-tie went the other way (measured: median 2e-7, max
    # 4e-2 at T=64); a wrong layer order or a missing residual gives O(1)
    assert np.median(e) < 1e-4 and e.max() < 0.25


def _report_free_run(xg, free):
    toks, x_free = free
    e = rel_l2(xg[toks], x_free)
    print(f"free-running oracle through 40 layers, tokens {list(toks)}: relative L2 {e}")
    # each layer is checked teacher-forced above; free running, the binary64
    # oracle and the binary32 device drift apart through 40 rounds of Q8_0
    # requantisation and routing (measured 4e-2 and 6e-2 at T=64); the bound
    # only catches gross errors (a skipped layer or norm gives O(1))
    assert np.all(np.isfinite(x_free)) and e.max() < 0.25


def test_stack40_decode_batch_t64():
    x0, xg, layers, free, x2 = _run_stack(64, n_check=2)
    _check_one_call(x0, xg, x2, layers)
    _report_free_run(xg, free)


def test_stack40_prefill_t4096():
    x0, xg, layers, free, x2 = _run_stack(4096, n_check=2)
    _check_one_call(x0, xg, x2, layers)
    _report_free_run(xg, free)
