"""Brute-force binary64 references used to pin the oracle on tiny shapes.

These dequantise everything to binary64 with numpy and run dense matmuls, the
plain definition of the layer without any per-block integer arithmetic.  They
are independent code: they never call the oracle.
"""
import numpy as np


def dequant_q4_0(blocks: np.ndarray) -> np.ndarray:
    """[..., nb, 18] uint8 -> [..., nb*32] float64 (low nibbles first, then high)."""
    blocks = np.asarray(blocks, dtype=np.uint8)
    d = blocks[..., 0:2].copy().view("<f2")[..., 0].astype(np.float64)
    qs = blocks[..., 2:18]
    vals = np.concatenate([(qs & 0x0F), (qs >> 4)], axis=-1).astype(np.float64) - 8.0
    w = vals * d[..., None]
    return w.reshape(blocks.shape[:-2] + (blocks.shape[-2] * 32,))


def dequant_q8_0(q: np.ndarray, d_bits: np.ndarray) -> np.ndarray:
    q = np.asarray(q, dtype=np.int8).astype(np.float64)
    d = np.asarray(d_bits, dtype=np.uint16).view(np.float16).astype(np.float64)
    return (q.reshape(q.shape[:-1] + (-1, 32)) * d[..., None]).reshape(q.shape)


def silu(g):
    g = np.asarray(g, dtype=np.float64)
    return g / (1.0 + np.exp(-g))
