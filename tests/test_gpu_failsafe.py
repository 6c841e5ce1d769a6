"""Failure detection without a GPU fault: a kernel waits on an mbarrier that
nothing arrives at, its bounded wait expires after a short limit, the device
error word reports it, and the context stays usable for normal work."""
import pytest
import torch

import mxfp8_block_scaled_fp8_b200 as fp8mm
from mxfp8_block_scaled_fp8_b200 import synthetic
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_and_reports():
    gu.require_gpu()
    assert fp8mm.last_device_error() == 0
    st = fp8mm.selftest_wait_timeout(2000)          # 2 ms limit
    assert st == fp8mm.fp8mm.FP8MM_ERR_DEVICE
    assert fp8mm.last_device_error() == 0           # the self-test cleared the word
    # the context is still good: a normal GEMM runs and is correct afterwards
    a, bt = synthetic.tiny()
    ga, gsa = fp8mm.fp8_quantize_rowwise(gu.to_dev(a))
    gb, gsb = fp8mm.fp8_quantize_rowwise(gu.to_dev(bt))
    c = fp8mm.fp8_gemm(ga, gb, gsa, gsb)
    torch.cuda.synchronize()
    assert torch.isfinite(c.float()).all()
    assert fp8mm.last_device_error() == 0
