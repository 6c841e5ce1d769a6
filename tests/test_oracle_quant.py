"""Pins for the oracle's two quantizers: invariants the amax/448 rule fixes
(page "从 DeepGEMM 到 vLLM", listing 3) and the MX block rule (32 elements per
UE8M0 scale, page "[sglang] FlashInfer v0.6.7 MXFP8 Gemm 통합", section 1),
checked against exact rational arithmetic done here, not by re-running the
oracle's formula."""
import json
import os
from fractions import Fraction

import numpy as np
import torch

from mxfp8_block_scaled_fp8_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


def _facts():
    with open(GOLDEN) as f:
        return json.load(f)


def _half_ulp_e4m3(a: float) -> float:
    """Half the E4M3 spacing at magnitude a (a <= 448)."""
    if a < 2.0 ** -6:
        return 2.0 ** -10
    e = int(np.floor(np.log2(a)))
    return 2.0 ** (e - 3) / 2


def _bits(t):
    return synthetic.bits(t)


def test_rowwise_invariants_random(orc):
    x = synthetic.random_bf16((64, 320), seed=11)
    x[3] *= 1e-30                                     # tiny row (scale stays normal fp32)
    x[5] *= 1e30                                      # huge row
    q, s = orc.quantize_rowwise(_bits(x))
    dec = orc.e4m3_decode_table()
    xf = x.float().numpy()
    for r in range(x.shape[0]):
        amax = np.abs(xf[r]).max()
        assert s[r] == np.float32(np.float64(amax) / _facts()["scale_rule_divisor"]["value"])
        d = dec[q[r]]
        assert np.abs(d).max() == 448.0               # the amax element maps to the max code
        # sign kept (incl. -0), error at most half an E4M3 spacing of x/s,
        # plus one fp32 rounding of the quotient
        assert np.all((q[r] >> 7) == np.signbit(xf[r]))
        quot = xf[r].astype(np.float64) / np.float64(s[r])
        for j in range(x.shape[1]):
            bound = _half_ulp_e4m3(min(abs(quot[j]), 448.0)) + abs(quot[j]) * 2.0 ** -23
            assert abs(d[j] - quot[j]) <= bound


def test_rowwise_special_rows(orc):
    x = torch.zeros((4, 64), dtype=torch.bfloat16)
    x[1] = 3.0
    x[2] = -0.5
    x[3, ::2] = -0.0
    q, s = orc.quantize_rowwise(_bits(x))
    assert s[0] == 1.0 and np.all(q[0] == 0x00)       # all-zero row: scale 1
    assert s[1] == np.float32(3.0 / 448.0) and np.all(q[1] == 0x7E)
    assert s[2] == np.float32(0.5 / 448.0) and np.all(q[2] == 0xFE)
    assert s[3] == 1.0 and np.all(q[3, ::2] == 0x80) and np.all(q[3, 1::2] == 0x00)


def test_rowwise_scale_fp32_division_equals_fp64_then_round():
    """The scale is amax/448 held in fp32.  For every bf16 amax the fp32
    quotient equals the fp64 quotient rounded to fp32 (no double-rounding
    case exists), so the kernel's fp32 division and the oracle agree."""
    bits = np.arange(0, 0x7F80, dtype=np.uint32).astype(np.uint16)  # positive finite bf16
    a = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).float()
    f32 = (a / torch.tensor(448.0, dtype=torch.float32)).numpy()
    f64 = (a.double() / 448.0).float().numpy()
    assert np.array_equal(f32.view(np.uint32), f64.view(np.uint32))


def test_rowwise_exact_quotients(orc):
    """Rows whose quotients x/s are exactly E4M3 values reproduce them."""
    vals = [448.0, 224.0, 1.0, -2.5, 0.015625, -0.001953125, 288.0, 0.0]
    x = torch.tensor([vals], dtype=torch.float32).to(torch.bfloat16)
    q, s = orc.quantize_rowwise(_bits(x))
    assert s[0] == 1.0
    dec = orc.e4m3_decode_table()
    assert list(dec[q[0]]) == vals


def test_mx_invariants_random(orc):
    x = synthetic.random_bf16((40, 256), seed=12, sigma=3.0)
    x[7, :32] *= 1e-35                                # a block that hits the low clamp
    x[9] *= 1e20
    q, sf = orc.mx_quantize(_bits(x))
    assert sf.shape == (40, 256 // _facts()["mx_elements_per_scale"]["value"])
    dec = orc.e4m3_decode_table()
    xf = x.float().numpy().astype(np.float64)
    for r in range(x.shape[0]):
        for b in range(sf.shape[1]):
            blk = xf[r, 32 * b:32 * b + 32]
            e = int(sf[r, b])
            amax = np.abs(blk).max()
            scale = Fraction(2) ** (e - 127)
            assert 0 <= e <= 254
            assert Fraction(float(amax)) <= 448 * scale          # never saturates
            if e > 0:
                assert Fraction(float(amax)) > 224 * scale       # smallest such scale
            d = dec[q[r, 32 * b:32 * b + 32]]
            for j in range(32):
                exact = Fraction(float(blk[j])) / scale          # exact scaled value
                err = abs(Fraction(float(d[j])) - exact)
                assert err <= Fraction(_half_ulp_e4m3(min(abs(float(exact)), 448.0)))
                assert (q[r, 32 * b + j] >> 7) == np.signbit(blk[j])


def test_mx_special_blocks(orc):
    x = torch.zeros((2, 128), dtype=torch.bfloat16)
    x[0, 32:64] = 448.0 * 2 ** -5                     # amax exactly 448 * 2^-5
    x[0, 64:96] = -3.0
    x[1, :32] = torch.linspace(-1, 1, 32)
    x[1, 96:128] = 1e-40                              # bf16 subnormal block
    q, sf = orc.mx_quantize(_bits(x))
    assert sf[0, 0] == 127 and np.all(q[0, :32] == 0)           # zero block: scale 1
    assert sf[0, 1] == 122 and np.all(q[0, 32:64] == 0x7E)      # maps to 448 exactly
    assert sf[0, 2] == 127 - 7 + 0                               # 3/448 -> ceil(log2) = -7
    dec = orc.e4m3_decode_table()
    assert np.all(dec[q[0, 64:96]] == -3.0 * 2 ** 7)             # 384, exactly representable
    assert sf[1, 0] == 119                                       # amax 1 -> 2^-8
    assert sf[1, 3] == 0                                         # low clamp


def test_quantizers_handle_real_workload_rows(orc):
    """A slice of the MX Q.K^T workload: the outlier rows get larger scales."""
    a, _ = synthetic.qk()
    q, sf = orc.mx_quantize(_bits(a[:64]))
    g = torch.Generator().manual_seed(1)
    assert sf.shape == (64, 128)
    assert sf.min() >= 100 and sf.max() <= 140
