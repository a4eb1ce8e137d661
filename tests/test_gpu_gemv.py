"""The W4A8 LM-head GEMV (one vocabulary-sized Q4_0 matrix) against the
oracle's W4A8 matrix-vector product of the same Q8_0 activations: the Q8_0
codes bit for bit, every output of sampled rows within 1e-5 of the row
scale (both sides sum exact per-block integer products; only the binary32
summation order differs)."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import quantized_moe_q4_b200 as m  # noqa: E402


def _matrix(seed, N, H):
    rng = np.random.Generator(np.random.PCG64(seed))
    return synth._q4_0_matrix(rng, N, H // 32)


@pytest.mark.parametrize("N,H,T", [(131072, 2048, 1), (131072, 2048, 5), (1000, 512, 8), (4096, 4096, 3),
                                   (64, 256, 2),
                                   # rows of 48, 56, 72, 80 blocks: chunks of 24, 8, 24, 16 blocks
                                   (700, 1536, 2), (300, 1792, 1), (520, 2304, 4), (128, 2560, 3)])
def test_gemv_matches_oracle(N, H, T):
    W = _matrix(N + H, N, H)
    x = np.random.default_rng(T).standard_normal((T, H)).astype(np.float32)
    y = m.moe_q4_gemv(torch.from_numpy(W).cuda(), torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    y = y.cpu().numpy()
    assert y.shape == (T, N) and np.all(np.isfinite(y))
    rows = np.unique(np.concatenate([[0, N - 1], np.random.default_rng(N).choice(N, min(N, 2000), replace=False)]))
    q, d, _ = oracle.quantize_q8_0(x)
    for t in range(T):
        ref = oracle.q4_matvec(W[rows], q[t], d[t])
        scale = max(float(np.sqrt(np.mean(ref.astype(np.float64) ** 2))), 1e-30)
        err = np.abs(y[t, rows].astype(np.float64) - ref) / np.maximum(np.abs(ref), scale)
        assert err.max() <= 1e-5, f"token {t}: worst {err.max():.2e}"
