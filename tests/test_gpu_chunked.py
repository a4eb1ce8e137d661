"""Chunked prefill (the prompt in several calls of C tokens) against the
oracle: every chunk is a layer call of its own, checked teacher-forced on
sampled tokens, and the chunked output agrees with the single-pass output
except where a last-bit difference between kernel families flipped a Q8_0
code of h."""
import numpy as np
import pytest
import torch

from gpu_helpers import rule13, run_forward, teacher_forced_check, workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import quantized_moe_q4_b200 as m  # noqa: E402


@pytest.mark.parametrize("C", [64, 200, 512])
def test_chunked_prefill_947(C):
    x, lw = workload("prefill_t947")
    T = x.shape[0]
    y_single = run_forward(lw, x, want_h=False)["y"]
    y_chunked = np.empty_like(y_single)
    rng = np.random.default_rng(C)
    for t0 in range(0, T, C):
        xc = x[t0:t0 + C]
        v = run_forward(lw, xc, want_h=False)
        toks = np.unique(np.concatenate([[0, xc.shape[0] - 1], rng.choice(xc.shape[0], 4, replace=False)]))
        teacher_forced_check(lw, xc, v, toks)
        y_chunked[t0:t0 + C] = v["y"]
    off = [t for t in range(T) if not rule13(y_chunked[t:t + 1], y_single[t:t + 1], 1e-3)[0]]
    assert len(off) <= T // 100, f"{len(off)} tokens differ between chunked and single-pass prefill"
