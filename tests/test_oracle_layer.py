"""Pins of the oracle's block dot products, projections, routing, permutation
and the whole MoE expert FFN layer (the grouped 4-bit GEMM and W4A8 kernels of
Methodologie 1 of the Dutch technical summary of "A 35B Hybrid-Attention
Mixture-of-Experts Model on a 6GB 2011 GPU").

Pins: a hand-worked block dot product (tests/golden/block_dot.txt), dense
binary64 dequantised matmuls (tests/bruteforce.py), numpy's stable sort and
softmax for routing, invariants of top-k and of the permutation, and the
degenerate cases E=1/k=1, all-zero weights, uniform logits, and a SwiGLU
gate driven far negative.
"""
import numpy as np
import pytest

import oracle
import synth
from bruteforce import dequant_q4_0, dequant_q8_0, silu
from golden_io import hexbytes, rows


def test_block_dot_golden():
    for hx, acts, I, dw16, da16, contrib in rows("block_dot.txt"):
        blk = np.frombuffer(hexbytes(hx), dtype=np.uint8)
        qa = np.array([int(v) for v in acts.split()], dtype=np.int8)
        assert qa.size == 32
        assert oracle.block_dot(blk, qa) == int(I)
        # the scaled contribution through a one-block matvec
        b = blk.copy()
        b[0:2] = np.frombuffer(int(dw16, 16).to_bytes(2, "little"), np.uint8)
        out = oracle.q4_matvec(b.reshape(1, 1, 18), qa, np.array([int(da16, 16)], np.uint16))
        assert float(out[0]) == float(contrib)


def test_block_dot_extremes():
    # all nibbles 0 (weight -8) against all q = 127 / -127: +-8*127*32
    blk = np.zeros(18, np.uint8)
    blk[0:2] = [0x00, 0x3C]
    assert oracle.block_dot(blk, np.full(32, 127, np.int8)) == -8 * 127 * 32
    assert oracle.block_dot(blk, np.full(32, -127, np.int8)) == 8 * 127 * 32
    blk[2:] = 0xFF  # weight 7
    assert oracle.block_dot(blk, np.full(32, -127, np.int8)) == -7 * 127 * 32


def test_block_dots_vs_dense_integer_dot():
    """The batched block dot (used to check the device's per-block sums in
    bulk) against numpy's integer dot of the dequantised nibbles: with the
    scale set to 1.0 a Q4_0 block dequantises to exactly nibble - 8."""
    rng = np.random.default_rng(21)
    n = 3000
    blocks = rng.integers(0, 256, size=(n, 18), dtype=np.uint8)
    blocks[:, 0:2] = [0x00, 0x3C]
    qa = rng.integers(-127, 128, size=(n, 32), dtype=np.int8)
    qa[0], blocks[0, 2:] = 127, 0x00                  # -8 * 127 * 32
    qa[1], blocks[1, 2:] = -127, 0xFF                 # 7 * -127 * 32
    w = dequant_q4_0(blocks.reshape(n, 1, 18)).reshape(n, 32)
    assert np.array_equal(w, np.rint(w)) and w.min() >= -8 and w.max() <= 7
    ref = np.einsum("ij,ij->i", w.astype(np.int64), qa.astype(np.int64))
    got = oracle.block_dots(blocks, qa)
    assert got.dtype == np.int32 and np.array_equal(got, ref)
    assert got[0] == -8 * 127 * 32 and got[1] == -7 * 127 * 32
    # the hand-worked block, inside a batch of shape [2, 1]
    for hx, acts, I, *_ in rows("block_dot.txt"):
        blk = np.frombuffer(hexbytes(hx), dtype=np.uint8)
        q = np.array([int(v) for v in acts.split()], dtype=np.int8)
        out = oracle.block_dots(np.stack([blk, blk])[:, None], np.stack([q, -q])[:, None])
        assert out.shape == (2, 1) and out[0, 0] == int(I) and out[1, 0] == -int(I)


@pytest.mark.parametrize("N,K", [(7, 64), (33, 256), (16, 512)])
def test_q4_matvec_vs_dense_binary64(N, K):
    rng = np.random.default_rng(N * K)
    x, layer = synth.random_layer(seed=N + K, H=K, F=32, E=1, k=1, shared=False)
    W = layer.w_gate[0][:N] if N <= 32 else np.concatenate([layer.w_gate[0]] * 2)[:N]
    xr = rng.standard_normal(K).astype(np.float32)
    qa, da, _ = oracle.quantize_q8_0(xr)
    got = oracle.q4_matvec(W, qa, da)
    ref = dequant_q4_0(W) @ dequant_q8_0(qa, da)
    # each term is exact in binary64; only summation order differs before the
    # final rounding to binary32
    assert np.allclose(got, ref, rtol=2 ** -23, atol=1e-30)
    assert np.all(np.abs(got - ref.astype(np.float32)) <= np.spacing(np.abs(ref).astype(np.float32)))


def test_router_logits_vs_numpy():
    x, layer = synth.random_layer(seed=4, H=96, F=32, E=12, k=3, shared=False, T=9)
    bias = np.linspace(-1, 1, 12).astype(np.float32)
    got = oracle.router_logits(x, layer.w_router, bias)
    ref = x.astype(np.float64) @ layer.w_router.astype(np.float64).T + bias
    assert np.allclose(got, ref.astype(np.float32), rtol=1e-6, atol=1e-7)
    # E x H is not square: a transposed operand cannot pass
    assert got.shape == (9, 12)


def test_topk_vs_numpy_stable_sort_and_softmax():
    rng = np.random.default_rng(8)
    T, E, k = 50, 20, 5
    logits = rng.standard_normal((T, E)).astype(np.float32)
    logits[3, :] = 0.25                           # all tied
    logits[4, 7] = logits[4, 2] = logits[4].max() + 1.0   # tie at the top
    idx, w = oracle.topk_softmax(logits, k)
    ref_idx = np.argsort(-logits, axis=1, kind="stable")[:, :k]
    assert np.array_equal(idx, ref_idx)
    assert list(idx[3]) == [0, 1, 2, 3, 4]
    assert list(idx[4][:2]) == [2, 7]
    sel = np.take_along_axis(logits, ref_idx, 1).astype(np.float64)
    ex = np.exp(sel - sel.max(axis=1, keepdims=True))
    ref_w = ex / ex.sum(axis=1, keepdims=True)
    assert np.allclose(w, ref_w, rtol=1e-6, atol=0)
    assert np.allclose(w.sum(axis=1, dtype=np.float64), 1.0, atol=1e-6)
    assert np.all(np.diff(w, axis=1) <= 0)
    for t in range(T):
        assert len(set(idx[t])) == k


def test_topk_brute_force_tiny():
    # every subset of size k of E=6: the chosen set maximises the sum of logits
    import itertools
    rng = np.random.default_rng(1)
    for _ in range(50):
        l = rng.standard_normal((1, 6)).astype(np.float32)
        idx, _ = oracle.topk_softmax(l, 3)
        best = max(itertools.combinations(range(6), 3), key=lambda s: sum(float(l[0, i]) for i in s))
        assert set(idx[0]) == set(best)


def test_uniform_logits_k_equals_e():
    E = 8
    logits = np.zeros((3, E), np.float32)
    idx, w = oracle.topk_softmax(logits, E)
    assert np.array_equal(idx, np.tile(np.arange(E), (3, 1)))
    assert np.all(w == np.float32(1.0 / E))


def test_permutation_invariants():
    rng = np.random.default_rng(2)
    T, k, E = 300, 6, 17
    logits = rng.standard_normal((T, E)).astype(np.float32)
    idx, _ = oracle.topk_softmax(logits, k)
    cnt, off, srt, pos = oracle.permute(idx, E)
    P = T * k
    assert np.array_equal(cnt, np.bincount(idx.ravel(), minlength=E))
    assert off[0] == 0 and off[-1] == P and np.array_equal(np.diff(off), cnt)
    assert np.array_equal(np.sort(srt), np.arange(P))                 # bijection
    assert np.array_equal(srt[pos], np.arange(P))                     # inverse
    assert np.array_equal(pos[srt], np.arange(P))
    flat = idx.ravel()
    for e in range(E):
        seg = srt[off[e]:off[e + 1]]
        assert np.all(flat[seg] == e)
        assert np.all(np.diff(seg) > 0)                               # stable: (t, j) order


def test_permutation_empty_and_single_expert():
    cnt, off, srt, pos = oracle.permute(np.zeros((0, 2), np.int32), 4)
    assert list(cnt) == [0, 0, 0, 0] and list(off) == [0, 0, 0, 0, 0]
    idx = np.array([[3], [3], [0]], np.int32)
    cnt, off, srt, pos = oracle.permute(idx, 4)
    assert list(cnt) == [1, 0, 0, 2] and list(srt) == [2, 0, 1] and list(pos) == [1, 2, 0]


# ---------------------------------------------------------------- layer


def _dense_reference(layer, x, y_dbg):
    """Binary64 dense reference of every stage, fed with the oracle's own
    routing and requantised intermediates (those are pinned separately)."""
    T, H = x.shape
    k = layer.top_k
    J = k + (1 if layer.has_shared else 0)
    g_ref = np.zeros((T, J, layer.ffn))
    u_ref = np.zeros_like(g_ref)
    o_ref = np.zeros((T, J, H))
    xq = dequant_q8_0(y_dbg["qa"], y_dbg["da"])
    for t in range(T):
        for j in range(J):
            if j < k:
                e = y_dbg["idx"][t, j]
                Wg, Wu, Wd = layer.w_gate[e], layer.w_up[e], layer.w_down[e]
            else:
                Wg, Wu, Wd = layer.sh_gate, layer.sh_up, layer.sh_down
            g_ref[t, j] = dequant_q4_0(Wg) @ xq[t]
            u_ref[t, j] = dequant_q4_0(Wu) @ xq[t]
            o_ref[t, j] = dequant_q4_0(Wd) @ dequant_q8_0(y_dbg["hq"][t, j], y_dbg["dh"][t, j])
    return g_ref, u_ref, o_ref


@pytest.mark.parametrize("shared", [False, True])
def test_layer_stages_vs_dense_binary64(shared):
    x, layer = synth.random_layer(seed=21, H=64, F=64, E=4, k=2, shared=shared, T=3)
    y, dbg = oracle.moe_forward(layer, x, debug=True)
    g_ref, u_ref, o_ref = _dense_reference(layer, x, dbg)
    f32 = lambda a: a.astype(np.float32)
    sp = lambda a: np.spacing(np.abs(f32(a)))
    assert np.all(np.abs(dbg["g"] - f32(g_ref)) <= sp(g_ref))
    assert np.all(np.abs(dbg["u"] - f32(u_ref)) <= sp(u_ref))
    assert np.all(np.abs(dbg["o"] - f32(o_ref)) <= sp(o_ref))
    # SwiGLU then requantisation: the requantised value reconstructs h to half a step
    h_ref = silu(dbg["g"].astype(np.float64)) * dbg["u"]
    assert np.allclose(dbg["h"], h_ref, rtol=2 ** -23, atol=0)
    hd = dequant_q8_0(dbg["hq"], dbg["dh"])
    step = dbg["dh"].view(np.float16).astype(np.float64)
    # |q*d16 - h| <= d32/2 + 127*|d16 - d32|, and |d16 - d32| <= d32 * 2^-11
    bound = step[..., None] * (0.5 + 127 * 2.0 ** -11) * 1.001 + 1e-12
    assert np.all(np.abs(hd - dbg["h"]).reshape(*hd.shape[:-1], -1, 32) <= bound)
    # combine: routed outputs weighted by w, shared weight 1
    wts = np.concatenate([dbg["w"], np.ones((3, 1), np.float32)], axis=1)[:, : o_ref.shape[1]]
    y_ref = np.einsum("tj,tjh->th", wts.astype(np.float64), dbg["o"].astype(np.float64))
    assert np.allclose(y, y_ref, rtol=1e-6, atol=1e-6)
    # routing is the oracle's own top-k of its own logits
    idx2, w2 = oracle.topk_softmax(dbg["logits"], layer.top_k)
    assert np.array_equal(idx2, dbg["idx"]) and np.array_equal(w2, dbg["w"])


def test_dense_single_expert_reduces_to_dense_w4a8_ffn():
    # E=1, k=1, no shared expert: one dense FFN with routing weight exactly 1
    x, layer = synth.random_layer(seed=5, H=128, F=96, E=1, k=1, shared=False, T=4)
    y, dbg = oracle.moe_forward(layer, x, debug=True)
    assert np.all(dbg["w"] == 1.0) and np.all(dbg["idx"] == 0)
    xq = dequant_q8_0(dbg["qa"], dbg["da"])
    g = xq @ dequant_q4_0(layer.w_gate[0]).T
    u = xq @ dequant_q4_0(layer.w_up[0]).T
    h = silu(g.astype(np.float32)) * u.astype(np.float32)
    hq_d = dequant_q8_0(dbg["hq"][:, 0], dbg["dh"][:, 0])
    # requantisation error bound then the down projection
    assert np.allclose(hq_d, h, atol=float(np.abs(h).max()) / 127.0 * 0.51)
    y_ref = hq_d @ dequant_q4_0(layer.w_down[0]).T
    assert np.allclose(y, y_ref, rtol=1e-6, atol=1e-6)


def test_all_zero_weights_give_zero_output():
    x, layer = synth.random_layer(seed=6, H=64, F=32, E=3, k=2, shared=True, T=5)
    for w in (layer.w_gate, layer.w_up, layer.w_down, layer.sh_gate, layer.sh_up, layer.sh_down):
        w[..., 2:] = 0x88        # every nibble 8 -> weight 0
    y = oracle.moe_forward(layer, x)
    assert np.all(y == 0.0)


def test_only_up_or_gate_zero_gives_zero():
    for which in ("gate", "up"):
        x, layer = synth.random_layer(seed=7, H=64, F=32, E=2, k=1, shared=False, T=3)
        getattr(layer, "w_" + which)[..., 2:] = 0x88
        assert np.all(oracle.moe_forward(layer, x) == 0.0)


def test_swiglu_gate_far_negative_silences_the_expert():
    # gate rows give g << 0 (silu(g) ~ 0) while up gives u > 0: h must vanish.
    # Swapping the roles of gate and up (silu(u)*g) would give |h| ~ |g|.
    H, F = 64, 32
    # 127/128 quantises exactly: d = 1/128 (a binary16 value), q = 127
    x = np.full((1, H), 127.0 / 128.0, np.float32)
    _, layer = synth.random_layer(seed=9, H=H, F=F, E=1, k=1, shared=False)
    layer.w_gate[...] = 0
    layer.w_gate[..., 0:2] = np.frombuffer(np.float16(1.0).tobytes(), np.uint8)
    layer.w_gate[..., 2:] = 0x00          # weight -8 -> g = -8*64*127/128 = -508
    layer.w_up[...] = 0
    layer.w_up[..., 0:2] = np.frombuffer(np.float16(1.0).tobytes(), np.uint8)
    layer.w_up[..., 2:] = 0x99            # weight +1 -> u = 64*127/128 = 63.5
    y, dbg = oracle.moe_forward(layer, x, debug=True)
    assert np.all(dbg["g"] == -508.0) and np.all(dbg["u"] == 63.5)
    assert np.all(dbg["h"] == 0.0)          # silu(-508) = -508/(1+e^508) underflows binary32
    assert np.all(y == 0.0)
    # the opposite sign: g = 7*63.5 = 444.5, silu(g) = g up to e^-444: h = g*u exactly in binary32
    layer.w_gate[..., 2:] = 0xFF          # weight +7
    y, dbg = oracle.moe_forward(layer, x, debug=True)
    assert np.all(dbg["g"] == 444.5)
    assert np.all(dbg["h"] == np.float32(444.5 * 63.5))


def test_teacher_forcing_reproduces_free_run():
    x, layer = synth.random_layer(seed=12, H=64, F=64, E=5, k=2, shared=True, T=6)
    y, dbg = oracle.moe_forward(layer, x, debug=True)
    y2 = oracle.moe_forward(layer, x, forced_idx=dbg["idx"], forced_w=dbg["w"],
                            forced_hq=dbg["hq"], forced_dh=dbg["dh"])
    assert np.array_equal(y, y2)
    # a different forced routing changes the output
    idx = (dbg["idx"] + 1) % 5
    y3 = oracle.moe_forward(layer, x, forced_idx=idx, forced_w=dbg["w"])
    assert not np.array_equal(y, y3)


def test_router_bias_shifts_selection():
    x, layer = synth.random_layer(seed=13, H=64, F=32, E=6, k=2, shared=False, T=20)
    layer.router_bias = np.array([0, 0, 0, 0, 0, 100.0], np.float32)
    _, dbg = oracle.moe_forward(layer, x, debug=True)
    assert np.all(dbg["idx"][:, 0] == 5)


def test_zero_tokens():
    x, layer = synth.random_layer(seed=14, H=64, F=32, E=3, k=2, shared=True, T=1)
    y = oracle.moe_forward(layer, np.zeros((0, 64), np.float32))
    assert y.shape == (0, 64)


def test_zipf_bias_recipe():
    b = synth.zipf_bias(128, 1.2)
    p = np.exp(b.astype(np.float64))
    assert abs(p.sum() - 1) < 1e-5
    assert abs(p[0] - 0.270) < 0.005 and abs(p[-1] - 8.0e-4) < 0.5e-4
    assert np.all(np.diff(b) < 0)
