"""Seeded synthetic inputs for the 4-bit MoE expert FFN.

This module only draws random numbers and lays them out in the Q4_0 byte
format; it holds none of the method's arithmetic.  The CUDA path's tests and
benchmark and the CPU oracle's tests all take their inputs from here.

Recipe (numpy PCG64, one generator per layer, fixed draw order):
  1. x      [T, H] fp32 ~ N(0, 1)
  2. Wr     [E, H] fp32 ~ N(0, 0.02)
  3. bias   [E] fp32: none, or log p_e for a Zipf(s) expert popularity
            p_r = r^-s / sum_{r'<=E} r'^-s, assigned by expert index
            (expert 0 the most popular); deterministic, no draw
  4. for each expert in order, for gate, up, down in that order:
        scales  fp16(|N(0,1)| * 0.02), rounded to nearest binary16
        nibbles 16 uniform random bytes per block (so every nibble is
                uniform over 0..15)
  5. the shared expert last, in the same way.
A Q4_0 block is 18 bytes: the binary16 scale little endian, then the 16
nibble bytes.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

QK = 32
Q4_BYTES = 18


@dataclass
class LayerWeights:
    hidden: int
    ffn: int
    n_experts: int
    top_k: int
    w_router: np.ndarray                 # [E, H] fp32
    router_bias: Optional[np.ndarray]    # [E] fp32 or None
    w_gate: np.ndarray                   # [E, F, H/32, 18] uint8
    w_up: np.ndarray                     # [E, F, H/32, 18] uint8
    w_down: np.ndarray                   # [E, H, F/32, 18] uint8
    sh_gate: Optional[np.ndarray] = None  # [F, H/32, 18] uint8
    sh_up: Optional[np.ndarray] = None
    sh_down: Optional[np.ndarray] = None  # [H, F/32, 18] uint8

    @property
    def has_shared(self) -> bool:
        return self.sh_gate is not None


# Workloads: the shapes and distributions the benchmark and the parity tests use.
WORKLOADS = {
    # small single layer the oracle finishes in well under a second
    "tiny_t16": dict(T=16, H=512, F=256, E=16, k=4, shared=False, zipf=None),
    # decode: one token per call, 1000 distinct tokens timed back to back
    "decode_t1": dict(T=1, H=2048, F=512, E=128, k=8, shared=True, zipf=None, tokens=1000),
    # single-pass prefill of a 947-token prompt
    "prefill_t947": dict(T=947, H=2048, F=512, E=128, k=8, shared=True, zipf=None),
    # 40-layer stack, batched decode (T=64) and prefill (T=4096)
    "stack40": dict(T=64, T_prefill=4096, H=2048, F=512, E=128, k=8, shared=True, zipf=None, layers=40),
    # load-skewed prefill: Zipf(1.2) expert popularity through the router bias
    "zipf_t16384": dict(T=16384, H=2048, F=512, E=128, k=8, shared=True, zipf=1.2),
}


def _q4_0_matrix(rng: np.random.Generator, rows: int, nblocks: int) -> np.ndarray:
    n = rows * nblocks
    scales = (np.abs(rng.standard_normal(n, dtype=np.float32)) * np.float32(0.02)).astype("<f2")
    nib = rng.integers(0, 256, size=(n, 16), dtype=np.uint8)
    out = np.empty((n, Q4_BYTES), dtype=np.uint8)
    out[:, 0:2] = scales.view(np.uint8).reshape(n, 2)
    out[:, 2:] = nib
    return out.reshape(rows, nblocks, Q4_BYTES)


def zipf_bias(n_experts: int, s: float) -> np.ndarray:
    r = np.arange(1, n_experts + 1, dtype=np.float64)
    p = r ** (-s)
    p /= p.sum()
    return np.log(p).astype(np.float32)


def make_layer(rng: np.random.Generator, H: int, F: int, E: int, k: int, shared: bool,
               zipf: Optional[float] = None) -> LayerWeights:
    """Router and expert weights, drawn in the recipe's order (after x)."""
    Wr = rng.standard_normal((E, H), dtype=np.float32) * np.float32(0.02)
    bias = zipf_bias(E, zipf) if zipf else None
    wg = np.empty((E, F, H // QK, Q4_BYTES), np.uint8)
    wu = np.empty_like(wg)
    wd = np.empty((E, H, F // QK, Q4_BYTES), np.uint8)
    for e in range(E):
        wg[e] = _q4_0_matrix(rng, F, H // QK)
        wu[e] = _q4_0_matrix(rng, F, H // QK)
        wd[e] = _q4_0_matrix(rng, H, F // QK)
    sg = su = sd = None
    if shared:
        sg = _q4_0_matrix(rng, F, H // QK)
        su = _q4_0_matrix(rng, F, H // QK)
        sd = _q4_0_matrix(rng, H, F // QK)
    return LayerWeights(H, F, E, k, Wr, bias, wg, wu, wd, sg, su, sd)


def make_inputs(T: int, H: int, F: int, E: int, k: int, shared: bool, zipf: Optional[float] = None,
                seed: int = 0):
    """(x [T,H] fp32, LayerWeights) for one layer, all from one PCG64(seed)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal((T, H), dtype=np.float32)
    layer = make_layer(rng, H, F, E, k, shared, zipf)
    return x, layer


def workload_inputs(name: str, seed: int = 0, T: Optional[int] = None):
    """Inputs of a named workload; `T` overrides the token count (decode_t1:
    the number of distinct tokens, default 1000)."""
    c = WORKLOADS[name]
    if T is None:
        T = c.get("tokens", c["T"])
    return make_inputs(T, c["H"], c["F"], c["E"], c["k"], c["shared"], c["zipf"], seed)


def stack_layer(layer_index: int, H: int, F: int, E: int, k: int, shared: bool, seed: int = 0):
    """Layer `layer_index` of a multi-layer stack: its own generator spawned
    from (seed, layer_index), so layers are independent of one another."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 1000 + layer_index])))
    return make_layer(rng, H, F, E, k, shared, None)


def stack_inputs(T: int, H: int, seed: int = 0) -> np.ndarray:
    """Input activations x [T,H] of a multi-layer stack (first draw of
    PCG64(seed); the layers come from stack_layer)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.standard_normal((T, H), dtype=np.float32)


def random_layer(seed: int, H: int, F: int, E: int, k: int, shared: bool, zipf=None, T: int = 1):
    """Small random case for property tests: same recipe, any shape."""
    return make_inputs(T, H, F, E, k, shared, zipf, seed)
