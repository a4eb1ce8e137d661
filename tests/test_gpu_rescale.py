"""The epilogue-rescale measurement kernel (moe_q4_rescale_ceiling): it must do
the arithmetic it claims to time.  Every accumulator chunk c of a thread
holds the integer 1 + c (as fp32 for binary16 operands, as ACC_BIAS + 1 + c
for int8 ones), and the block scales are fixed fp32 patterns, so the first
thread's checksum after `iters` stages is a closed-form sum; both operand
types must give it (the int8 path's bias removal is exact), within fp32
accumulation rounding of the binary64 value."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import quantized_moe_q4_b200 as m  # noqa: E402


def _expected_checksum(iters):
    i = np.arange(4 * 4 * 32)
    da = (np.float32(1.0) + (i & 63).astype(np.float32) * np.float32(1.0 / 1024.0)).astype(np.float64)
    dw = float(np.float32(1.0 / 4096.0))      # row 0: index a multiple of 128, so (i & 31) = 0
    total = 0.0
    for it in range(iters):
        sc = it & 3
        for qc in range(8):                   # 4 blocks x 2 chunks of 16 columns
            kb, hf = qc >> 1, qc & 1
            base = (sc * 4 + kb) * 32 + 16 * hf
            total += (1 + qc) * dw * da[base:base + 16].sum()
    return total


@pytest.mark.parametrize("int8_operands", [False, True])
@pytest.mark.parametrize("iters", [1, 5, 64])
def test_rescale_ceiling_checksum(int8_operands, iters):
    sink = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
    n = m.moe_q4_rescale_ceiling(int8_operands, iters, sink)
    torch.cuda.synchronize()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert n == sms * 16 * 32 * 128 * iters
    want = _expected_checksum(iters)
    got = float(sink.item())
    assert abs(got - want) <= 1e-5 * abs(want), (got, want)
