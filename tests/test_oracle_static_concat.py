"""Pins for the oracle's per-tensor scale, static-scale quantizer and key
concatenation, each against something other than itself: the already pinned
per-row quantizer and encoder, closed forms, and brute-force loops.

Pages: "FP8 推理基础设施（五）：从 DeepGEMM 到 vLLM", listing 3 (one scale per
tensor, max|x| / 448); "[flashinfer] FlashInfer, FP8 지원으로 장문 컨텍스트 추론
성능을 극적으로 향상시키다", 코드 분석 items 1 and 3 (nope and rope parts of a key
concatenated per head)."""
import numpy as np
import pytest
import torch

import oracle as orc
from mxfp8_block_scaled_fp8_b200 import synthetic


def _bits(x: torch.Tensor) -> np.ndarray:
    return synthetic.bits(x)


def test_tensor_scale_is_the_largest_row_scale():
    # fp32 rounding is monotone, so fp32(max_r amax_r / 448) = max_r fp32(amax_r / 448)
    for seed in range(4):
        x = synthetic.random_bf16((37, 96), seed=seed, sigma=3.0)
        x[seed] *= 50.0
        _, s_rows = orc.quantize_rowwise(_bits(x))
        assert orc.tensor_scale(_bits(x)) == s_rows.max()


@pytest.mark.parametrize("j", [-30, -3, 0, 5, 60])
def test_tensor_scale_closed_forms(j):
    x = torch.zeros((4, 64), dtype=torch.bfloat16)
    x[2, 7] = -448.0 * 2.0 ** j          # amax = 448 * 2^j  ->  s = 2^j exactly
    x[1, 3] = 448.0 * 2.0 ** (j - 1)
    assert orc.tensor_scale(_bits(x)) == np.float32(2.0 ** j)
    assert orc.tensor_scale(_bits(torch.zeros((3, 32), dtype=torch.bfloat16))) == np.float32(1.0)


def _all_bf16_up_to(limit: float) -> torch.Tensor:
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    v = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
    f = v.float()
    return v[torch.isfinite(f) & (f.abs() <= limit)]


def test_static_with_unit_scale_is_the_encoder():
    v = _all_bf16_up_to(448.0)
    n = v.numel() // 64 * 64
    x = v[:n].reshape(-1, 64).contiguous()
    q = orc.quantize_static(_bits(x), 1.0)
    expect = orc.e4m3_encode(x.double().numpy().ravel()).reshape(x.shape)
    assert np.array_equal(q, expect)


@pytest.mark.parametrize("j", [-8, -1, 3, 20])
def test_static_with_power_of_two_scale_is_exact_scaling(j):
    x = synthetic.random_bf16((19, 160), seed=j + 100, sigma=2.0 ** j)
    q = orc.quantize_static(_bits(x), 2.0 ** j)
    expect = orc.e4m3_encode((x.double() * 2.0 ** -j).numpy().ravel()).reshape(x.shape)
    assert np.array_equal(q, expect)


def test_static_with_the_row_scale_is_the_row_quantizer():
    x = synthetic.random_bf16((1, 4096), seed=9, sigma=0.7)
    q_row, s_row = orc.quantize_rowwise(_bits(x))
    assert np.array_equal(orc.quantize_static(_bits(x), s_row[0]), q_row)


def _concat_loops(nope: np.ndarray, rope: np.ndarray) -> np.ndarray:
    T, H, dn = nope.shape
    dr = rope.shape[2]
    out = np.zeros((T, H, dn + dr), dtype=nope.dtype)
    for t in range(T):
        for h in range(H):
            for i in range(dn):
                out[t, h, i] = nope[t, h, i]
            for i in range(dr):
                out[t, h, dn + i] = rope[t, 0 if rope.shape[1] == 1 else h, i]
    return out


@pytest.mark.parametrize("rope_heads", [1, 3])
def test_concat_matches_loops(rope_heads):
    g = np.random.default_rng(5)
    nope = g.integers(0, 256, size=(4, 3, 16), dtype=np.uint8)
    rope = g.integers(0, 256, size=(4, rope_heads, 8), dtype=np.uint8)
    assert np.array_equal(orc.concat_mla_k(nope, rope), _concat_loops(nope, rope))
    n16 = g.integers(0, 65536, size=(2, 5, 8), dtype=np.uint16)
    r16 = g.integers(0, 65536, size=(2, rope_heads if rope_heads == 1 else 5, 8), dtype=np.uint16)
    assert np.array_equal(orc.concat_mla_k(n16, r16), _concat_loops(n16, r16))


def test_concat_written_out_example():
    # one token, two heads, nope 2, rope 1 (broadcast): [[a b r], [c d r]]
    nope = np.array([[[1, 2], [3, 4]]], dtype=np.uint8)
    rope = np.array([[[9]]], dtype=np.uint8)
    assert orc.concat_mla_k(nope, rope).tolist() == [[[1, 2, 9], [3, 4, 9]]]
