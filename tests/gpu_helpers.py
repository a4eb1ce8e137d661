"""Shared helpers of the GPU parity tests: run the CUDA path through the C-ABI
binding, map its slot-ordered intermediates back to (token, slot) pairs, and
check them against the oracle."""
import numpy as np
import torch

import oracle
import synth

_CACHE = {}


def workload(name, seed=0, T=None):
    key = (name, seed, T)
    if key not in _CACHE:
        _CACHE[key] = synth.workload_inputs(name, seed=seed, T=T)
    return _CACHE[key]


def device_layer(lw):
    import quantized_moe_q4_b200 as m
    key = ("dev", id(lw))
    if key not in _CACHE:
        _CACHE[key] = (lw, m.Layer.from_host(lw))
    return _CACHE[key][1]


def run_forward(lw, x_np, path=0, want_h=True, L=None):
    """One forward on the device; returns numpy copies of y, h and the
    workspace intermediates (slot-ordered).  `L`: the layer's device copy
    (default: a cached upload of lw)."""
    import quantized_moe_q4_b200 as m
    L = device_layer(lw) if L is None else L
    x = torch.from_numpy(np.ascontiguousarray(x_np)).cuda()
    T = x.shape[0]
    y = torch.empty_like(x)
    ws = m.alloc_workspace(m.moe_q4_ffn_workspace_bytes(L, T))
    slots = T * lw.top_k + (T if lw.sh_gate is not None else 0)
    h = torch.full((slots, lw.ffn), float("nan"), device="cuda") if want_h else None
    m.moe_q4_ffn_forward_debug(L, x, y, ws, h_out=h, path=path)
    torch.cuda.synchronize()
    v = {k: t.cpu().numpy() for k, t in m.workspace_views(L, T, ws).items()}
    v["y"] = y.cpu().numpy()
    if want_h:
        v["h"] = h.cpu().numpy()
    return v


def pairs_from_slots(lw, T, v, arr):
    """[slots, ...] slot-ordered array -> [T, k+S, ...] in (token, j) order."""
    k = lw.top_k
    S = 1 if lw.sh_gate is not None else 0
    P = T * k
    out = np.empty((T, k + S) + arr.shape[1:], arr.dtype)
    pos = v["pos"].reshape(T, k)
    out[:, :k] = arr[pos]
    if S:
        out[:, k] = arr[P:P + T]
    return out


def rule13(y, y_ref, rel=1e-3):
    """Per element |y - y_ref| <= rel * max(|y_ref|, rms of its row).
    Returns (ok, worst ratio)."""
    y = np.asarray(y, np.float64)
    r = np.asarray(y_ref, np.float64)
    rms = np.sqrt(np.mean(r * r, axis=-1, keepdims=True))
    scale = np.maximum(np.abs(r), rms)
    scale = np.where(scale > 0, scale, 1e-30)
    ratio = np.abs(y - r) / scale
    return bool(np.all(ratio <= rel)), float(ratio.max()) if ratio.size else 0.0


def teacher_forced_check(lw, x_np, v, tokens, rel=1e-3):
    """Oracle with the GPU's routing (idx, w) and requantised SwiGLU output
    (hq, dh) on the given tokens; y and h are compared, hq must be the
    oracle's Q8_0 of the GPU's own h bit for bit."""
    T = x_np.shape[0]
    tokens = np.asarray(tokens)
    hq_p = pairs_from_slots(lw, T, v, v["hq"])[tokens]
    dh_p = pairs_from_slots(lw, T, v, v["dh"].view(np.uint16))[tokens]
    y_ref, dbg = oracle.moe_forward(lw, x_np[tokens], forced_idx=v["topk_idx"][tokens],
                                    forced_w=v["topk_w"][tokens], forced_hq=hq_p, forced_dh=dh_p, debug=True)
    ok, worst = rule13(v["y"][tokens], y_ref, rel)
    assert ok, f"y differs from the teacher-forced oracle: worst ratio {worst:.3e}"
    if "h" in v:
        h_p = pairs_from_slots(lw, T, v, v["h"])[tokens]
        ok_h, worst_h = rule13(h_p, dbg["h"], 1e-4)
        assert ok_h, f"SwiGLU output h differs: worst ratio {worst_h:.3e}"
        q, d, _ = oracle.quantize_q8_0(h_p)
        assert np.array_equal(q, hq_p), "requantised h differs from the oracle's Q8_0 of the GPU's h"
        assert np.array_equal(d, dh_p), "binary16 scales of requantised h differ"
    # activation quantisation is bit-exact
    assert np.array_equal(v["qa"][tokens], dbg["qa"])
    assert np.array_equal(v["da"][tokens].view(np.uint16), dbg["da"])
    return worst


def check_routing(lw, x_np, v, rel_logit=2e-5):
    """GPU logits vs the oracle's; GPU top-k == the oracle's top-k of the GPU's
    own logits (bit for bit); weights vs the oracle's softmax."""
    T = x_np.shape[0]
    ref = oracle.router_logits(x_np, lw.w_router, lw.router_bias)
    scale = np.maximum(np.abs(ref).max(axis=1, keepdims=True), 1e-6)
    err = np.abs(v["logits"] - ref) / scale
    assert err.max() <= rel_logit, f"router logits: max relative error {err.max():.2e}"
    idx, w = oracle.topk_softmax(v["logits"], lw.top_k)
    assert np.array_equal(v["topk_idx"], idx), "top-k indices differ given identical logits"
    assert np.allclose(v["topk_w"], w, rtol=2e-6, atol=1e-7)
    return ref


def check_permutation(lw, v):
    T = v["topk_idx"].shape[0]
    cnt, off, srt, pos = oracle.permute(v["topk_idx"], lw.n_experts)
    E = lw.n_experts
    S = 1 if lw.sh_gate is not None else 0
    assert np.array_equal(v["cnt"][:E], cnt)
    assert v["cnt"][E] == S * T
    assert np.array_equal(v["off"][:E + 1], off)
    assert v["off"][E + 1] == T * lw.top_k + S * T
    assert np.array_equal(v["sorted"], srt)
    assert np.array_equal(v["pos"], pos)


def near_tie_tokens(lw, x_np, v):
    """Tokens whose free-running routing differs from the oracle's and whether
    each difference is a near-tie: the oracle's logit gap at the changed
    positions is within twice the largest logit error."""
    ref = oracle.router_logits(x_np, lw.w_router, lw.router_bias)
    idx_ref, _ = oracle.topk_softmax(ref, lw.top_k)
    bad = []
    for t in np.nonzero(np.any(idx_ref != v["topk_idx"], axis=1))[0]:
        dl = float(np.abs(v["logits"][t] - ref[t]).max())
        srt = np.sort(ref[t])[::-1]
        gaps = np.abs(np.diff(srt[:lw.top_k + 1]))
        bad.append((int(t), bool(gaps.min() <= 2 * dl + 1e-12)))
    return bad
