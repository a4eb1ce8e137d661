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


# Two runs of the T = 1 path add the (k+S) x F/32 partial sums of an output
# element of y (144 for the 2048/512 layer with 8 routed experts and a shared
# one) in different orders.  Recursive summation of n binary32 terms errs by
# at most (n - 1) u sum|t| (u = 2^-24), so two orders differ by at most
# 2 (n - 1) u sum|t|: about 1.6e-4 of rule13's scale when sum|t| is ten times
# the row's rms; rounding errors of random sign stay near sqrt(n) u of it
# (about 1e-6).  The run-to-run comparisons take 1e-5, between the two.
ORDER_REL = 1e-5


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


def expected_block_dots(lw, T, v, down, g, rb, R):
    """The oracle's per-block integer dot products of one row block of one
    expert group, in the layout of moe_q4_debug.block_dots_out: [slot of the
    group][row][block], from the device's own Q8_0 activations (bit-exact with
    the oracle's, checked separately) and the layer's Q4_0 rows."""
    k, E = lw.top_k, lw.n_experts
    P = T * k
    s0, s1 = int(v["off"][g]), int(v["off"][g + 1])
    slots = np.arange(s0, s1)
    if down:
        acts = v["hq"][slots]
        W = lw.sh_down if g == E else lw.w_down[g]
        Wr = W[rb * R:(rb + 1) * R]
    else:
        tok = (v["sorted"][slots] // k) if g < E else (slots - P)
        acts = v["qa"][tok]
        Wg = lw.sh_gate if g == E else lw.w_gate[g]
        Wu = lw.sh_up if g == E else lw.w_up[g]
        half = R // 2
        Wr = np.concatenate([Wg[rb * half:(rb + 1) * half], Wu[rb * half:(rb + 1) * half]])
    c, nb = len(slots), Wr.shape[1]
    blocks = np.broadcast_to(Wr[None], (c, R, nb, 18))
    a = np.broadcast_to(acts.reshape(c, 1, nb, 32), (c, R, nb, 32))
    return oracle.block_dots(blocks, a)


def tile_boundary_tokens(lw, T, v, groups, tile):
    """Tokens of the first and the last slot of every `tile`-slot tile of the
    given expert groups (group E: the shared expert, slot P + t = token t)."""
    k, E = lw.top_k, lw.n_experts
    P = T * k
    toks = []
    for g in groups:
        s0, s1 = int(v["off"][g]), int(v["off"][g + 1])
        if s1 <= s0:
            continue
        firsts = np.arange(s0, s1, tile)
        lasts = np.minimum(firsts + tile - 1, s1 - 1)
        sl = np.unique(np.concatenate([firsts, lasts]))
        toks.append((v["sorted"][sl] // k) if g < E else (sl - P))
    return np.unique(np.concatenate(toks)) if toks else np.zeros(0, np.int64)


def free_running_report(lw, x_np, v, tokens):
    """The device's free-running output against the independent oracle (its
    own routing and requantisation) on `tokens`:
      identical   tokens whose top-k matches the oracle's (same order);
      near_tie    tokens whose top-k differs, each at a near-tie (the
                  oracle's logit gap at a changed position within twice the
                  largest logit difference);
      other       tokens whose top-k differs beyond a near-tie (must be 0);
      requant     identical tokens whose requantised SwiGLU output (a code
                  or a binary16 scale of h) differs from the oracle's: the
                  binary32 h of the device and the binary64-then-binary32 h
                  of the oracle straddle a rounding boundary;
      row_err     the largest norm-wise row error |y - y_ref| / |y_ref| over
                  the identical tokens without a requantisation difference;
      requant_row_err  the same over the tokens with one;
      within_1e3  the fraction of identical tokens with row error <= 1e-3;
      flips       Q8_0 codes of h that differ by one step (identical tokens),
      big_flips   codes that differ by more (must be 0), scale_diffs the
                  binary16 scales of h that differ."""
    tokens = np.asarray(tokens)
    T = x_np.shape[0]
    y_ref, dbg = oracle.moe_forward(lw, x_np[tokens], debug=True)
    idx_dev = v["topk_idx"][tokens]
    same = np.all(idx_dev == dbg["idx"], axis=1)
    ties = dict(near_tie_tokens(lw, x_np, v))
    diff_toks = tokens[~same]
    near = sum(1 for t in diff_toks if ties.get(int(t), False))
    y = v["y"][tokens].astype(np.float64)
    r = y_ref.astype(np.float64)
    row_err = np.linalg.norm(y - r, axis=1) / np.maximum(np.linalg.norm(r, axis=1), 1e-30)
    hq_dev = pairs_from_slots(lw, T, v, v["hq"])[tokens]
    dh_dev = pairs_from_slots(lw, T, v, v["dh"].view(np.uint16))[tokens]
    dq = np.abs(hq_dev.astype(np.int32) - dbg["hq"].astype(np.int32))
    req = same & ((dq.reshape(len(tokens), -1).max(axis=1) > 0) |
                  np.any((dh_dev != dbg["dh"]).reshape(len(tokens), -1), axis=1))
    exact = same & ~req
    dqs = dq[same]
    return dict(tokens=int(len(tokens)), identical=int(same.sum()), near_tie=int(near),
                other=int(len(diff_toks) - near), requant=int(req.sum()),
                row_err=float(row_err[exact].max()) if exact.any() else 0.0,
                row_err_median=float(np.median(row_err[exact])) if exact.any() else 0.0,
                requant_row_err=float(row_err[req].max()) if req.any() else 0.0,
                within_1e3=float(np.mean(row_err[same] <= 1e-3)) if same.any() else 1.0,
                flips=int(np.count_nonzero(dqs == 1)), big_flips=int(np.count_nonzero(dqs > 1)),
                scale_diffs=int(np.count_nonzero(dh_dev[same] != dbg["dh"][same])))
