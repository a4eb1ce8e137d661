"""The host SIMD W4A8 baseline against the oracle: per-block integer dot
products bit for bit (including the extreme blocks), the layer within the
free-running tolerance on the tiny and decode workloads."""
import numpy as np

import cpu_simd
import oracle
from gpu_helpers import rule13, workload


def test_block_dots_bit_exact():
    rng = np.random.default_rng(5)
    n = 2048
    blocks = rng.integers(0, 256, size=(n, 18), dtype=np.uint8)
    qa = rng.integers(-127, 128, size=(n, 32), dtype=np.int8)
    blocks[0, 2:] = 0x00
    qa[0] = 127
    blocks[1, 2:] = 0xFF
    qa[1] = -127
    got = cpu_simd.block_dots(blocks, qa)
    ref = np.array([oracle.block_dot(blocks[i], qa[i]) for i in range(n)], np.int32)
    assert np.array_equal(got, ref)
    assert got[0] == -8 * 127 * 32 and got[1] == -7 * 127 * 32


def test_layer_matches_oracle_tiny():
    x, lw = workload("tiny_t16")
    ok, worst = rule13(cpu_simd.moe_forward(lw, x), oracle.moe_forward(lw, x), 1e-2)
    assert ok, worst


def test_layer_matches_oracle_decode_tokens():
    x, lw = workload("decode_t1", T=1000)
    xs = x[:6]
    ok, worst = rule13(cpu_simd.moe_forward(lw, xs), oracle.moe_forward(lw, xs), 1e-2)
    assert ok, worst
