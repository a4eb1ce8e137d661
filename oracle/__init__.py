"""CPU oracle of the 4-bit MoE expert FFN (numpy front end over plain C).

TEST INFRASTRUCTURE ONLY: the tests, the package entry module's smoke check and
the benchmark's CPU-baseline leg may import this package; the product path
(`quantized_moe_q4_b200`) never does, and the two share no code.

What it computes follows the Dutch technical summary of "A 35B Hybrid-Attention
Mixture-of-Experts Model on a 6GB 2011 GPU: Hand-Written 4-bit CUDA Inference
for Fermi" (gist.science/nl/paper/2606.24031), Methodologie 1 (grouped 4-bit
GEMM for the MoE, W4A8 integer decode kernel) and Methodologie 2 (group-wise
symmetric Q4_0-family weights, 8-bit activations, 128 experts per layer).
The block formats and routing rules the page leaves open are fixed in
`moe_q4_oracle.c`'s header.

Parity pins: every function here is pinned by tests under `tests/` marked
`not gpu` (hand-worked blocks in `tests/golden/`, binary16 conversion against
numpy, brute-force binary64 dequantised matmuls, routing and permutation
invariants, degenerate cases).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

from . import build as _build

QK = 32
Q4_BYTES = 18

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64, i32 = ctypes.c_int64, ctypes.c_int
        lib.orc_half_to_double.argtypes = [ctypes.c_uint16]
        lib.orc_half_to_double.restype = ctypes.c_double
        lib.orc_float_to_half_rne.argtypes = [ctypes.c_float]
        lib.orc_float_to_half_rne.restype = ctypes.c_uint16
        lib.orc_round_half_away.argtypes = [ctypes.c_float]
        lib.orc_round_half_away.restype = ctypes.c_int
        lib.orc_quantize_q8_0.argtypes = [P, i64, P, P]
        lib.orc_quantize_q8_0.restype = ctypes.c_int
        lib.orc_q4_0_dequant.argtypes = [P, i64, P]
        lib.orc_block_dot.argtypes = [P, P]
        lib.orc_block_dot.restype = ctypes.c_int32
        lib.orc_block_dots.argtypes = [P, i64, P, P]
        lib.orc_q4_matvec.argtypes = [P, i32, i32, P, P, P]
        lib.orc_router_logits.argtypes = [P, i64, i32, P, P, i32, P]
        lib.orc_topk_softmax.argtypes = [P, i64, i32, i32, P, P]
        lib.orc_permute.argtypes = [P, i64, i32, i32, P, P, P, P]
        lib.orc_moe_forward.argtypes = [P, P, i64, P, P, P, P, P, P]
        lib.orc_moe_forward.restype = ctypes.c_int
        lib.orc_rmsnorm.argtypes = [P, i64, i32, ctypes.c_float, P]
        lib.orc_residual_add.argtypes = [P, P, i64]
        lib.orc_set_threads.argtypes = [i32]
        lib.orc_set_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def set_threads(n: int = 0) -> int:
    """Set (n>0) and return the OpenMP thread count of the oracle's token loops."""
    return _load().orc_set_threads(int(n))


# ---------------------------------------------------------------- scalars


def half_to_double(bits) -> np.ndarray:
    lib = _load()
    b = np.asarray(bits, dtype=np.uint16)
    return np.array([lib.orc_half_to_double(int(v)) for v in b.ravel()], dtype=np.float64).reshape(b.shape)


def float_to_half_rne(x) -> np.ndarray:
    lib = _load()
    f = np.asarray(x, dtype=np.float32)
    return np.array([lib.orc_float_to_half_rne(float(v)) for v in f.ravel()], dtype=np.uint16).reshape(f.shape)


def round_half_away(x) -> np.ndarray:
    lib = _load()
    f = np.asarray(x, dtype=np.float32)
    return np.array([lib.orc_round_half_away(float(v)) for v in f.ravel()], dtype=np.int64).reshape(f.shape)


# ---------------------------------------------------------------- blocks


def quantize_q8_0(x: np.ndarray):
    """Q8_0 of x (last dim a multiple of 32) -> (q int8 same shape, d uint16 [..., n/32], overflow flag)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    n = x.size
    assert x.shape[-1] % QK == 0
    q = np.empty(x.shape, dtype=np.int8)
    d = np.empty(x.shape[:-1] + (x.shape[-1] // QK,), dtype=np.uint16)
    ov = _load().orc_quantize_q8_0(_ptr(x), n, _ptr(q), _ptr(d))
    return q, d, bool(ov)


def q4_0_dequant(blocks: np.ndarray) -> np.ndarray:
    """Dequantise Q4_0 blocks [..., nb, 18] -> float64 [..., nb*32]."""
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
    assert blocks.shape[-1] == Q4_BYTES
    nb = blocks.size // Q4_BYTES
    out = np.empty(blocks.shape[:-2] + (blocks.shape[-2] * QK,), dtype=np.float64)
    _load().orc_q4_0_dequant(_ptr(blocks), nb, _ptr(out))
    return out


def block_dot(blk: np.ndarray, qa: np.ndarray) -> int:
    blk = np.ascontiguousarray(blk, dtype=np.uint8).reshape(Q4_BYTES)
    qa = np.ascontiguousarray(qa, dtype=np.int8).reshape(QK)
    return int(_load().orc_block_dot(_ptr(blk), _ptr(qa)))


def block_dots(blocks: np.ndarray, qa: np.ndarray) -> np.ndarray:
    """block_dot over many blocks: blocks [..., 18] uint8 and qa [..., 32]
    int8 with the same leading shape -> int32 [...]."""
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
    qa = np.ascontiguousarray(qa, dtype=np.int8)
    assert blocks.shape[-1] == Q4_BYTES and qa.shape[-1] == QK and blocks.shape[:-1] == qa.shape[:-1]
    out = np.empty(blocks.shape[:-1], dtype=np.int32)
    _load().orc_block_dots(_ptr(blocks), out.size, _ptr(qa), _ptr(out))
    return out


def q4_matvec(W: np.ndarray, qa: np.ndarray, da: np.ndarray) -> np.ndarray:
    """W [N, K/32, 18] Q4_0, one Q8_0 row (qa [K], da [K/32]) -> fp32 [N]."""
    W = np.ascontiguousarray(W, dtype=np.uint8)
    N, nb = W.shape[0], W.shape[1]
    out = np.empty(N, dtype=np.float32)
    _load().orc_q4_matvec(_ptr(W), N, nb * QK, _ptr(np.ascontiguousarray(qa, np.int8)),
                          _ptr(np.ascontiguousarray(da, np.uint16)), _ptr(out))
    return out


# ---------------------------------------------------------------- routing


def router_logits(x: np.ndarray, w_router: np.ndarray, bias: Optional[np.ndarray] = None) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    Wr = np.ascontiguousarray(w_router, dtype=np.float32)
    T, H = x.shape
    E = Wr.shape[0]
    out = np.empty((T, E), dtype=np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    _load().orc_router_logits(_ptr(x), T, H, _ptr(Wr), _ptr(b), E, _ptr(out))
    return out


def topk_softmax(logits: np.ndarray, k: int):
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float32)
    _load().orc_topk_softmax(_ptr(logits), T, E, k, _ptr(idx), _ptr(w))
    return idx, w


def permute(idx: np.ndarray, n_experts: int):
    """Stable counting sort of the T*k (token, slot) pairs by expert.

    Returns cnt [E], off [E+1], sorted [T*k], pos [T*k]."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    P = T * k
    cnt = np.empty(n_experts, np.int32)
    off = np.empty(n_experts + 1, np.int32)
    srt = np.empty(P, np.int32)
    pos = np.empty(P, np.int32)
    _load().orc_permute(_ptr(idx), T, k, n_experts, _ptr(cnt), _ptr(off), _ptr(srt), _ptr(pos))
    return cnt, off, srt, pos


# ---------------------------------------------------------------- layer


class _OrcLayer(ctypes.Structure):
    _fields_ = [
        ("hidden", ctypes.c_int32), ("ffn", ctypes.c_int32), ("n_experts", ctypes.c_int32),
        ("top_k", ctypes.c_int32), ("has_shared", ctypes.c_int32),
        ("w_router", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
        ("w_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p),
        ("sh_gate", ctypes.c_void_p), ("sh_up", ctypes.c_void_p), ("sh_down", ctypes.c_void_p),
    ]


class _OrcDebug(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("logits", "idx", "w", "qa", "da", "g", "u", "h", "hq", "dh", "o", "overflow")]


def moe_forward(layer, x: np.ndarray, *, forced_idx=None, forced_w=None, forced_hq=None,
                forced_dh=None, debug: bool = False):
    """The MoE expert FFN layer for T tokens.

    `layer` has numpy attributes w_router [E,H] f32, router_bias [E] f32 or None,
    w_gate/w_up [E,F,H/32,18] u8, w_down [E,H,F/32,18] u8, sh_gate/sh_up [F,H/32,18]
    and sh_down [H,F/32,18] (or None), and ints hidden, ffn, n_experts, top_k.
    Teacher forcing: forced_idx/forced_w [T,k] replace routing; forced_hq
    [T,k+S,F] / forced_dh [T,k+S,F/32] replace the requantised SwiGLU output
    (slot k = shared expert).  Returns y [T,H] fp32, or (y, dict) with debug.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    T, H = x.shape
    F, E, k = layer.ffn, layer.n_experts, layer.top_k
    S = 1 if layer.sh_gate is not None else 0
    J = k + S
    keep = []

    def c(a, dt):
        if a is None:
            return None
        a = np.ascontiguousarray(a, dtype=dt)
        keep.append(a)
        return a

    L = _OrcLayer(H, F, E, k, S,
                  _ptr(c(layer.w_router, np.float32)), _ptr(c(layer.router_bias, np.float32)),
                  _ptr(c(layer.w_gate, np.uint8)), _ptr(c(layer.w_up, np.uint8)),
                  _ptr(c(layer.w_down, np.uint8)),
                  _ptr(c(layer.sh_gate, np.uint8)), _ptr(c(layer.sh_up, np.uint8)),
                  _ptr(c(layer.sh_down, np.uint8)))
    y = np.empty((T, H), dtype=np.float32)
    dbg = None
    arrays = {}
    if debug:
        arrays = dict(
            logits=np.zeros((T, E), np.float32), idx=np.zeros((T, k), np.int32),
            w=np.zeros((T, k), np.float32), qa=np.zeros((T, H), np.int8),
            da=np.zeros((T, H // QK), np.uint16), g=np.zeros((T, J, F), np.float32),
            u=np.zeros((T, J, F), np.float32), h=np.zeros((T, J, F), np.float32),
            hq=np.zeros((T, J, F), np.int8), dh=np.zeros((T, J, F // QK), np.uint16),
            o=np.zeros((T, J, H), np.float32), overflow=np.zeros(1, np.int32))
        dbg = _OrcDebug(**{n: _ptr(a) for n, a in arrays.items()})
    rc = _load().orc_moe_forward(
        ctypes.byref(L), _ptr(x), T, _ptr(y),
        _ptr(c(forced_idx, np.int32)), _ptr(c(forced_w, np.float32)),
        _ptr(c(forced_hq, np.int8)), _ptr(c(forced_dh, np.uint16)),
        ctypes.byref(dbg) if dbg is not None else None)
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (rc={rc})")
    if debug:
        if forced_idx is not None:
            arrays["logits"] = None
        return y, arrays
    return y


# ---------------------------------------------------------------- stack glue


def rmsnorm(x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """Unit-gain RMSNorm of each row (the stack's reading of the inter-layer
    glue): mean of squares in binary64, xn = binary32(x / sqrt(mean + eps))."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    T, H = x.shape
    out = np.empty_like(x)
    _load().orc_rmsnorm(_ptr(x), T, H, float(eps), _ptr(out))
    return out


def residual_add(x: np.ndarray, y: np.ndarray) -> np.ndarray:
    """binary32(x + y), the exact sum rounded once."""
    out = np.array(x, dtype=np.float32, order="C", copy=True)
    y = np.ascontiguousarray(y, dtype=np.float32)
    assert y.shape == out.shape
    _load().orc_residual_add(_ptr(out), _ptr(y), out.size)
    return out


def stack_forward(layers, x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """x_{l+1} = x_l + MoE_l(RMSNorm(x_l)) through `layers` (free running)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    for lw in layers:
        x = residual_add(x, moe_forward(lw, rmsnorm(x, eps)))
    return x
