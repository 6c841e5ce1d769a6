"""FP8 key assembly for multi-head latent attention (concat_mla_k) and the
FP8 KV-cache quantizer, against the CPU oracle, bit for bit (page
"[flashinfer] FlashInfer, FP8 지원으로 장문 컨텍스트 추론 성능을 극적으로
향상시키다", 코드 분석 items 1, 3 and 5: E4M3 / E5M2 and 16-bit inputs, bit-exact
tests)."""
import numpy as np
import pytest
import torch

import mxfp8_block_scaled_fp8_b200 as fp8mm
from mxfp8_block_scaled_fp8_b200 import synthetic
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    gu.require_gpu()


def _bytes(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(0, 256, shape, generator=g, dtype=torch.int32).to(torch.uint8)


@pytest.mark.parametrize("rope_heads", [1, "H"])
@pytest.mark.parametrize("T,H", [(1, 1), (37, 16), (300, 128)])
def test_concat_fp8_bytes(T, H, rope_heads):
    import oracle as orc
    rh = H if rope_heads == "H" else 1
    nope = _bytes((T, H, 128), T + H)
    rope = _bytes((T, rh, 64), T * 3 + H)
    out = fp8mm.concat_mla_k(nope.cuda().view(torch.float8_e4m3fn), rope.cuda().view(torch.float8_e4m3fn))
    torch.cuda.synchronize()
    assert out.dtype == torch.float8_e4m3fn
    assert np.array_equal(out.view(torch.uint8).cpu().numpy(), orc.concat_mla_k(nope.numpy(), rope.numpy()))


def test_concat_e5m2_and_bf16():
    import oracle as orc
    nope = _bytes((9, 4, 128), 1)
    rope = _bytes((9, 1, 64), 2)
    out = fp8mm.concat_mla_k(nope.cuda().view(torch.float8_e5m2), rope.cuda().view(torch.float8_e5m2))
    assert np.array_equal(out.view(torch.uint8).cpu().numpy(), orc.concat_mla_k(nope.numpy(), rope.numpy()))
    n16 = synthetic.random_bf16((11, 8, 128), seed=3)
    r16 = synthetic.random_bf16((11, 1, 64), seed=4)
    out = fp8mm.concat_mla_k(n16.cuda(), r16.cuda())
    torch.cuda.synchronize()
    ref = orc.concat_mla_k(n16.view(torch.int16).numpy(), r16.view(torch.int16).numpy())
    assert np.array_equal(out.cpu().view(torch.int16).numpy(), ref)


def test_concat_strided_inputs_and_output():
    """k_nope as a slice of a wider per-head buffer, k_rope a slice of a wider
    per-token row, and the output a slice of a larger cache."""
    import oracle as orc
    T, H = 23, 12
    big = _bytes((T, H, 256), 7)
    ropebig = _bytes((T, 1, 96), 8)
    nope, rope = big[:, :, 64:192], ropebig[:, :, 16:80]
    cache = torch.zeros((T + 2, H, 224), dtype=torch.uint8, device="cuda")
    out = cache[1:T + 1, :, :192]
    fp8mm.concat_mla_k(big.cuda()[:, :, 64:192], ropebig.cuda()[:, :, 16:80], out=out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), orc.concat_mla_k(nope.numpy(), rope.numpy()))
    assert not cache[0].any() and not cache[T + 1].any() and not cache[:, :, 192:].any()


def test_concat_degenerate_and_errors():
    empty = torch.empty((0, 4, 128), dtype=torch.uint8, device="cuda")
    out = fp8mm.concat_mla_k(empty, torch.empty((0, 1, 64), dtype=torch.uint8, device="cuda"))
    assert out.shape == (0, 4, 192)
    with pytest.raises(fp8mm.Fp8mmError):                       # 120-byte rows are not 16-byte multiples
        fp8mm.concat_mla_k(torch.zeros((2, 2, 120), dtype=torch.uint8, device="cuda"),
                           torch.zeros((2, 1, 64), dtype=torch.uint8, device="cuda"))
    nope = torch.zeros((4, 2, 129), dtype=torch.uint8, device="cuda")[:, :, 1:]   # misaligned base
    with pytest.raises(fp8mm.Fp8mmError):
        fp8mm.concat_mla_k(nope, torch.zeros((4, 1, 64), dtype=torch.uint8, device="cuda"))


def test_fp8_kv_cache_quantize_then_concat():
    """The KV-cache path: bf16 nope and rope parts quantized with their
    per-tensor scales, then assembled; equals the oracle doing the same."""
    import oracle as orc
    T, H = 64, 16
    nope = synthetic.random_bf16((T * H, 128), seed=31, sigma=0.5)
    rope = synthetic.random_bf16((T, 64), seed=32, sigma=2.0)
    s_n = fp8mm.fp8_tensor_scale(gu.to_dev(nope))
    s_r = fp8mm.fp8_tensor_scale(gu.to_dev(rope))
    qn = fp8mm.fp8_quantize_static(gu.to_dev(nope), s_n)
    qr = fp8mm.fp8_quantize_static(gu.to_dev(rope), s_r)
    k = fp8mm.concat_mla_k(qn.view(T, H, 128), qr.view(T, 1, 64))
    torch.cuda.synchronize()
    qn_ref = orc.quantize_static(synthetic.bits(nope), orc.tensor_scale(synthetic.bits(nope)))
    qr_ref = orc.quantize_static(synthetic.bits(rope), orc.tensor_scale(synthetic.bits(rope)))
    ref = orc.concat_mla_k(qn_ref.reshape(T, H, 128), qr_ref.reshape(T, 1, 64))
    assert np.array_equal(k.cpu().numpy(), ref)
