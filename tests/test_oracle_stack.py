"""Pins of the oracle's inter-layer glue (unit-gain RMSNorm, residual add)
and of the multi-layer driver, each against a fact fixed independently of
the oracle's own code."""
import numpy as np

import oracle
import synth


def test_rmsnorm_one_hot_row_is_sqrt_h():
    # a row with one nonzero entry a: mean of squares a^2/H, so with eps = 0
    # the entry becomes sign(a) * sqrt(H) and the rest stay 0
    H = 64
    x = np.zeros((3, H), np.float32)
    x[0, 5] = 3.0
    x[1, 0] = -0.125
    x[2, 63] = 1e-20
    xn = oracle.rmsnorm(x, eps=0.0)
    assert xn[0, 5] == 8.0 and xn[1, 0] == -8.0 and xn[2, 63] == 8.0
    assert np.count_nonzero(xn) == 3


def test_rmsnorm_power_of_two_scaling_is_exact():
    # scaling a row by 4^k scales the mean of squares by 16^k and the rms by
    # 4^k exactly, so with eps = 0 the output is identical bit for bit
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 256)).astype(np.float32)
    a = oracle.rmsnorm(x, eps=0.0)
    for s in (4.0, 1.0 / 16.0, 1024.0):
        assert np.array_equal(oracle.rmsnorm(x * np.float32(s), eps=0.0), a)


def test_rmsnorm_output_has_unit_rms_and_eps_matters_only_for_tiny_rows():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((4, 2048)).astype(np.float32)
    xn = oracle.rmsnorm(x, eps=1e-6).astype(np.float64)
    assert np.allclose(np.sqrt(np.mean(xn * xn, axis=1)), 1.0, atol=1e-6)
    # a row of 1e-4 (mean square 1e-8, far below eps) comes out at about
    # 1e-4 / sqrt(1e-6) = 0.1 rather than 1
    tiny = np.full((1, 16), 1e-4, np.float32)
    v = oracle.rmsnorm(tiny, eps=1e-6)[0, 0]
    assert abs(v - 1e-4 / np.sqrt(1e-6 + 1e-8)) < 1e-6


def test_residual_add_is_one_ieee_rounding():
    # numpy's float32 addition is the IEEE single-precision sum
    rng = np.random.default_rng(2)
    x = rng.standard_normal(1000).astype(np.float32) * np.float32(1e3)
    y = rng.standard_normal(1000).astype(np.float32) * np.float32(1e-3)
    assert np.array_equal(oracle.residual_add(x, y), x + y)


def test_stack_of_zero_layers_is_identity():
    # all-8 nibbles make every weight 0, so every MoE output is exactly 0 and
    # x_{l+1} = x_l through the whole stack
    x, lw = synth.random_layer(seed=5, H=256, F=256, E=4, k=2, shared=True, T=3)
    for a in (lw.w_gate, lw.w_up, lw.w_down, lw.sh_gate, lw.sh_up, lw.sh_down):
        a[..., 2:] = 0x88
    out = oracle.stack_forward([lw, lw, lw], x)
    assert np.array_equal(out, x)


def test_stack_layer_generator_is_deterministic_and_layers_differ():
    a = synth.stack_layer(0, H=256, F=256, E=4, k=2, shared=True)
    b = synth.stack_layer(0, H=256, F=256, E=4, k=2, shared=True)
    c = synth.stack_layer(1, H=256, F=256, E=4, k=2, shared=True)
    assert np.array_equal(a.w_gate, b.w_gate) and not np.array_equal(a.w_gate, c.w_gate)


def test_stack_stays_bounded_over_many_layers():
    # with the normalisation every layer sees unit-rms input, so 12 layers of
    # the tiny shape keep x finite and its rms within a modest factor
    rng = np.random.default_rng(3)
    x = rng.standard_normal((2, 512)).astype(np.float32)
    layers = [synth.stack_layer(i, H=512, F=256, E=16, k=4, shared=False) for i in range(12)]
    out = oracle.stack_forward(layers, x)
    assert np.all(np.isfinite(out))
    r0 = np.sqrt(np.mean(x.astype(np.float64) ** 2))
    r1 = np.sqrt(np.mean(out.astype(np.float64) ** 2))
    assert r1 < 100 * r0
