"""The small-M scale layout (the use_8x4_sf_layout option of the mm_mxfp8 call,
page "[sglang] FlashInfer v0.6.7 MXFP8 Gemm 통합", section 2): the quantizer
writing it must give the oracle's codes and exponents bit for bit, with the
padding bytes zero, and the small-M GEMM reading it must give exactly the
result it gives from the 128-row chunk layout, within the bar of the oracle."""
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


def sf8x4_canonical(sf: np.ndarray, rows: int, k: int) -> np.ndarray:
    """Read the small-M layout into canonical [rows, k/32], from the layout
    formula written out here (atoms of 8 rows x 4 blocks, K-group major)."""
    rows8 = -(-rows // 8) * 8
    r = np.arange(rows)[:, None]
    b = np.arange(k // 32)[None, :]
    return sf[((b // 4) * (rows8 // 8) + r // 8) * 32 + (r % 8) * 4 + b % 4]


@pytest.mark.parametrize("rows,k", [(1, 4096), (5, 512), (8, 14336), (9, 4096), (17, 4128), (33, 1056),
                                    (64, 14336), (200, 256)])
def test_quantizer_8x4_bit_exact(rows, k):
    import oracle as orc
    x = synthetic.random_bf16((rows, k), seed=rows * 13 + k, sigma=2.0)
    if rows > 2:
        x[1] = 0.0                                             # zero row: exponent 127
        x[2, :32] *= 1e-37                                     # a block at the low clamp
    q_ref, sf_ref = orc.mx_quantize(synthetic.bits(x))
    xd = gu.to_dev(x)
    q, sf = fp8mm.mxfp8_quantize_8x4(xd)
    q128, _ = fp8mm.mxfp8_quantize(xd)
    torch.cuda.synchronize()
    sf = sf.cpu().numpy()
    assert sf.size == fp8mm.sf8x4_bytes(rows, k)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert torch.equal(q, q128)
    assert np.array_equal(sf8x4_canonical(sf, rows, k), sf_ref)
    written = np.zeros(sf.size, dtype=bool)
    r = np.arange(rows)[:, None]
    b = np.arange(k // 32)[None, :]
    written[np.array([fp8mm.sf8x4_offset(rows, k, int(i), int(j)) for i, j in
                      zip(np.broadcast_to(r, (rows, k // 32)).ravel(), np.broadcast_to(b, (rows, k // 32)).ravel())])] = True
    assert not sf[~written].any()                              # padding rows and blocks are zero


@pytest.mark.parametrize("name", ["up", "down", "qkv"])
@pytest.mark.parametrize("m", synthetic.DECODE_M + (16, 48))
def test_decode_gemm_reads_8x4_scales(name, m):
    """Every decode shape: identical bits from either scale layout with the
    same partition (tile-aligned ones reduced in clusters, the others through
    the workspace), and the bar against the oracle."""
    import oracle as orc
    ws_, xs = _decode()
    n, k = synthetic.DECODE_SHAPES[name]
    qw, sfw, gw, gsfw = ws_[name]
    x = xs[k][:m].contiguous()
    qx_ref, sfx_ref = orc.mx_quantize(synthetic.bits(x))
    xd = gu.to_dev(x)
    gx, gsf128 = fp8mm.mxfp8_quantize(xd)
    gx8, gsf8 = fp8mm.mxfp8_quantize_8x4(xd)
    wsp = torch.zeros(fp8mm.workspace_bytes(m, n, k), dtype=torch.uint8, device="cuda")
    c128 = fp8mm.mxfp8_gemm(gx, gsf128, gw, gsfw, workspace=wsp, weights_ready=True)
    c8 = fp8mm.mxfp8_gemm(gx8, gsf8, gw, gsfw, workspace=wsp, weights_ready=True, sf_a_8x4=True)
    torch.cuda.synchronize()
    assert torch.equal(c8, c128)
    c_ref, bound = orc.gemm_mx(qx_ref, sfx_ref, qw, sfw)
    gu.check_gemm(c8, c_ref, bound, f"8x4 scales {name} m={m}")
    assert fp8mm.last_device_error() == 0


@pytest.mark.parametrize("m,n,k,ctas", [(3, 200, 96, 0), (17, 130, 4128, 5), (40, 384, 896, 21), (64, 257, 1024, 3),
                                        (9, 1000, 512, 0)])
def test_8x4_ragged_and_partitions(m, n, k, ctas):
    import oracle as orc
    x = synthetic.random_bf16((m, k), seed=m * 5 + k)
    w = synthetic.random_bf16((n, k), seed=n * 3 + k, sigma=0.02)
    qx, sfx = orc.mx_quantize(synthetic.bits(x))
    qw, sfw = orc.mx_quantize(synthetic.bits(w))
    gw, gsfw = fp8mm.mxfp8_quantize(gu.to_dev(w))
    gx8, gsf8 = fp8mm.mxfp8_quantize_8x4(gu.to_dev(x))
    wsp = torch.zeros(max(fp8mm.workspace_bytes(m, n, k, ctas), 256), dtype=torch.uint8, device="cuda")
    c = fp8mm.mxfp8_gemm(gx8, gsf8, gw, gsfw, workspace=wsp, small_m_ctas=ctas, sf_a_8x4=True)
    torch.cuda.synchronize()
    c_ref, bound = orc.gemm_mx(qx, sfx, qw, sfw)
    gu.check_gemm(c, c_ref, bound, f"8x4 ragged {m}x{n}x{k} ctas={ctas}")


def test_8x4_only_for_the_small_m_kernel():
    gx8, gsf8 = fp8mm.mxfp8_quantize_8x4(gu.to_dev(synthetic.random_bf16((65, 256), seed=1)))
    gw, gsfw = fp8mm.mxfp8_quantize(gu.to_dev(synthetic.random_bf16((256, 256), seed=2)))
    with pytest.raises(fp8mm.Fp8mmError):                     # m > 64: tiled kernels read 128-row chunks
        fp8mm.mxfp8_gemm(gx8, gsf8, gw, gsfw, sf_a_8x4=True)
    with pytest.raises(fp8mm.Fp8mmError):
        fp8mm.mxfp8_gemm(gx8[:8], gsf8, gw, gsfw, sf_a_8x4=True, kernel=fp8mm.KERNEL_TILED)


_DECODE = None


def _decode():
    global _DECODE
    if _DECODE is None:
        import oracle as orc
        ws_, xs = synthetic.decode()
        out = {}
        for name, w in ws_.items():
            qw, sfw = orc.mx_quantize(synthetic.bits(w))
            gw, gsfw = fp8mm.mxfp8_quantize(gu.to_dev(w))
            out[name] = (qw, sfw, gw, gsfw)
        _DECODE = (out, xs)
    return _DECODE
