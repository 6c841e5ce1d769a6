"""Decode GEMM with the activation quantized inside the kernel
(mxfp8_quantize_gemm): the activation is quantized per call and the weights
once (page "[sglang] FlashInfer v0.6.7 MXFP8 Gemm 통합", section 2).  Its
output must equal, bit for bit, mxfp8_quantize followed by the small-M
mxfp8_gemm with the same stream-K partition (the quantized values and the
summation order are the same), and must meet the GEMM tolerance against the
CPU oracle on the quantized operands."""
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


@pytest.fixture(scope="module")
def weights():
    import oracle as orc
    ws, xs = synthetic.decode()
    out = {}
    for name, w in ws.items():
        qw, sfw = orc.mx_quantize(synthetic.bits(w))
        gw, gsfw = fp8mm.mxfp8_quantize(gu.to_dev(w))
        out[name] = (qw, sfw, gw, gsfw)
    return out, xs


def _ws(m, n, k, ctas=0):
    return torch.zeros(fp8mm.workspace_bytes(m, n, k, ctas), dtype=torch.uint8, device="cuda")


def _wsq(m, n, k, ctas=0):
    return torch.zeros(fp8mm.quantize_gemm_workspace_bytes(m, n, k, ctas), dtype=torch.uint8, device="cuda")


def _unfused(x_dev, gw, gsfw, ws, ctas=0):
    gx, gsfx = fp8mm.mxfp8_quantize(x_dev)
    return fp8mm.mxfp8_gemm(gx, gsfx, gw, gsfw, workspace=ws, kernel=fp8mm.KERNEL_SMALL_M, small_m_ctas=ctas)


@pytest.mark.parametrize("name", ["up", "down", "qkv"])
@pytest.mark.parametrize("m", synthetic.DECODE_M)
def test_fused_decode_sweep(weights, name, m):
    import oracle as orc
    ws_, xs = weights
    qw, sfw, gw, gsfw = ws_[name]
    n, k = synthetic.DECODE_SHAPES[name]
    x = xs[k][:m].contiguous()
    xd = gu.to_dev(x)
    ws = _wsq(m, n, k)
    c = fp8mm.mxfp8_quantize_gemm(xd, gw, gsfw, workspace=ws, weights_ready=True)
    c_ref_dev = _unfused(xd, gw, gsfw, _ws(m, n, k))
    torch.cuda.synchronize()
    assert torch.equal(c, c_ref_dev), f"fused {name} m={m} differs from quantize + GEMM"
    qx, sfx = orc.mx_quantize(synthetic.bits(x))
    c_ref, bound = orc.gemm_mx(qx, sfx, qw, sfw)
    gu.check_gemm(c, c_ref, bound, f"fused decode {name} m={m}")
    c2 = fp8mm.mxfp8_quantize_gemm(xd, gw, gsfw, workspace=ws, weights_ready=True)
    torch.cuda.synchronize()
    assert torch.equal(c, c2), "second call with the same workspace differs"


@pytest.mark.parametrize("m,n,k", [(1, 1, 32), (3, 200, 96), (8, 260, 4128), (9, 300, 4096), (16, 129, 8192),
                                   (17, 130, 4128),
                                   (33, 1000, 64), (49, 300, 160), (64, 384, 320)])
def test_fused_ragged_strided(m, n, k):
    """Ragged m, n and k (k a multiple of 32, not of 128), a row stride wider
    than k, with and without the stream-K split."""
    import oracle as orc
    base = synthetic.random_bf16((m, k + 40), seed=m * 7 + k)
    x = base[:, :k]
    w = synthetic.random_bf16((n, k), seed=n * 5 + k, sigma=0.02)
    qx, sfx = orc.mx_quantize(synthetic.bits(x.contiguous()))
    qw, sfw = orc.mx_quantize(synthetic.bits(w))
    c_ref, bound = orc.gemm_mx(qx, sfx, qw, sfw)
    xd = gu.to_dev(base)[:, :k]
    assert xd.stride(0) == k + 40
    gw, gsfw = fp8mm.mxfp8_quantize(gu.to_dev(w))
    for ctas in (0, 5):
        c = fp8mm.mxfp8_quantize_gemm(xd, gw, gsfw, workspace=_wsq(m, n, k, ctas), small_m_ctas=ctas)
        c_un = _unfused(xd.contiguous(), gw, gsfw, _ws(m, n, k, ctas), ctas)
        torch.cuda.synchronize()
        gu.check_gemm(c, c_ref, bound, f"fused ragged {m}x{n}x{k} ctas={ctas}")
        assert torch.equal(c, c_un), f"fused ragged {m}x{n}x{k} ctas={ctas} differs from quantize + GEMM"
    if m <= 8:                                                  # no workspace: one CTA per tile
        c = fp8mm.mxfp8_quantize_gemm(xd, gw, gsfw)
        torch.cuda.synchronize()
        gu.check_gemm(c, c_ref, bound, f"fused ragged {m}x{n}x{k} one CTA per tile")
    else:                                                       # the quantized activation needs the workspace
        with pytest.raises(fp8mm.Fp8mmError):
            fp8mm.mxfp8_quantize_gemm(xd, gw, gsfw)


@pytest.mark.parametrize("m", [5, 32])
@pytest.mark.parametrize("ctas", [1, 7, 300, 5000])
def test_fused_partitions(weights, ctas, m):
    ws_, xs = weights
    _, _, gw, gsfw = ws_["down"]
    n, k = synthetic.DECODE_SHAPES["down"]
    xd = gu.to_dev(xs[k][:m].contiguous())
    c = fp8mm.mxfp8_quantize_gemm(xd, gw, gsfw, workspace=_wsq(m, n, k, ctas), small_m_ctas=ctas)
    c_un = _unfused(xd, gw, gsfw, _ws(m, n, k, ctas), ctas)
    torch.cuda.synchronize()
    assert torch.equal(c, c_un)


def test_fused_reads_the_activation_after_the_preceding_kernel(weights):
    """The activation is rewritten by a kernel right before the call on the
    same stream; the fused kernel (launched to overlap its predecessor) must
    quantize the new values."""
    ws_, xs = weights
    _, _, gw, gsfw = ws_["up"]
    n, k = synthetic.DECODE_SHAPES["up"]
    x0 = gu.to_dev(xs[k][:8].contiguous())
    buf = torch.zeros_like(x0)
    ws = _wsq(8, n, k)
    fp8mm.mxfp8_quantize_gemm(buf, gw, gsfw, workspace=ws, weights_ready=True)      # warm, zeros
    for scale in (1.0, -2.0, 0.5):
        torch.mul(x0, scale, out=buf)                     # the preceding kernel writes the activation
        c = fp8mm.mxfp8_quantize_gemm(buf, gw, gsfw, workspace=ws, weights_ready=True)
        c_un = _unfused((x0 * scale).contiguous(), gw, gsfw, _ws(8, n, k))
        torch.cuda.synchronize()
        assert torch.equal(c, c_un), f"scale {scale}"


def test_fused_edge_values():
    """Zero rows, a zero block, bf16 subnormals and the largest bf16 values in
    the activation: the in-kernel quantizer must give mxfp8_quantize's codes."""
    import oracle as orc
    x = synthetic.random_bf16((12, 512), seed=9, sigma=3.0)
    x[0] = 0.0
    x[1, :32] = 0.0
    x[2] *= 1e-38
    x[3] = torch.finfo(torch.bfloat16).max
    x[3, 1::2] = -torch.finfo(torch.bfloat16).max
    x[4, 64:96] = 448.0 * 2 ** -9
    x[5] *= 1e30
    w = synthetic.random_bf16((256, 512), seed=10, sigma=0.02)
    gw, gsfw = fp8mm.mxfp8_quantize(gu.to_dev(w))
    xd = gu.to_dev(x)
    c = fp8mm.mxfp8_quantize_gemm(xd, gw, gsfw, workspace=_wsq(12, 256, 512))
    c_un = _unfused(xd, gw, gsfw, _ws(12, 256, 512))
    torch.cuda.synchronize()
    assert torch.equal(c, c_un)
    qx, sfx = orc.mx_quantize(synthetic.bits(x))
    qw, sfw = orc.mx_quantize(synthetic.bits(w))
    c_ref, bound = orc.gemm_mx(qx, sfx, qw, sfw)
    # rows whose products reach past the bf16 range (the +-bf16 max row) are
    # covered by the bit-for-bit comparison above only
    keep = bound.max(axis=1) < 1e37
    assert keep.sum() >= 10
    gu.check_gemm(c[torch.from_numpy(keep).cuda()], c_ref[keep], bound[keep], "fused edge values")


def test_fused_degenerate_and_errors(weights):
    ws_, xs = weights
    _, _, gw, gsfw = ws_["qkv"]
    n, k = synthetic.DECODE_SHAPES["qkv"]
    x = torch.empty((0, k), dtype=torch.bfloat16, device="cuda")
    c = fp8mm.mxfp8_quantize_gemm(x, gw, gsfw)
    assert c.shape == (0, n)
    x = gu.to_dev(synthetic.random_bf16((65, k), seed=65))
    with pytest.raises(fp8mm.Fp8mmError):
        fp8mm.mxfp8_quantize_gemm(x, gw, gsfw)                  # m > 64
    tiny_ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(fp8mm.Fp8mmError):                          # a split reduced through the workspace
        fp8mm.mxfp8_quantize_gemm(x[:8], gw, gsfw, workspace=tiny_ws, split_via_workspace=True)
    with pytest.raises(fp8mm.Fp8mmError):                          # 37 CTAs: not tile-aligned
        fp8mm.mxfp8_quantize_gemm(x[:8], gw, gsfw, workspace=tiny_ws, small_m_ctas=37)
    with pytest.raises(fp8mm.Fp8mmError):
        fp8mm.mxfp8_quantize_gemm(x[:8], gw, gsfw, kernel=fp8mm.KERNEL_TILED)
    with pytest.raises(fp8mm.Fp8mmError):                          # m > 8 without room for the activation
        fp8mm.mxfp8_quantize_gemm(x[:9], gw, gsfw, workspace=_ws(9, n, k))
    assert fp8mm.last_device_error() == 0
