"""Small-M (decode) MXFP8 kernel vs the CPU oracle: every M in {1, 8, 32, 64}
against the three Llama-3-8B-sized linears, with and without the stream-K
split, plus determinism and partition independence."""
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
def decode_data():
    import oracle as orc
    ws, xs = synthetic.decode()
    out = {}
    for name, w in ws.items():
        qw, sfw = orc.mx_quantize(synthetic.bits(w))
        gw, gsfw = fp8mm.mxfp8_quantize(gu.to_dev(w))
        out[name] = (qw, sfw, gw, gsfw)
    return out, xs


def _workspace(m, n, k, ctas=0):
    nbytes = fp8mm.workspace_bytes(m, n, k, ctas)
    return torch.zeros(nbytes, dtype=torch.uint8, device="cuda")


@pytest.mark.parametrize("name", ["up", "down", "qkv"])
@pytest.mark.parametrize("m", synthetic.DECODE_M)
def test_decode_sweep_stream_k(decode_data, name, m):
    import oracle as orc
    weights, xs = decode_data
    qw, sfw, gw, gsfw = weights[name]
    n, k = synthetic.DECODE_SHAPES[name]
    x = xs[k][:m].contiguous()
    qx, sfx = orc.mx_quantize(synthetic.bits(x))
    gx, gsfx = fp8mm.mxfp8_quantize(gu.to_dev(x))
    ws = _workspace(m, n, k)
    # the weights were quantized long before: they may be streamed while the
    # activation quantizer that precedes the GEMM is still running
    c = fp8mm.mxfp8_gemm(gx, gsfx, gw, gsfw, workspace=ws, weights_ready=True)
    torch.cuda.synchronize()
    c_ref, bound = orc.gemm_mx(qx, sfx, qw, sfw)
    gu.check_gemm(c, c_ref, bound, f"decode {name} m={m}")
    # counters are left at zero for the next call
    c2 = fp8mm.mxfp8_gemm(gx, gsfx, gw, gsfw, workspace=ws, weights_ready=True)
    torch.cuda.synchronize()
    assert torch.equal(c, c2), "second call with the same workspace differs"


@pytest.mark.parametrize("m", [1, 64])
def test_decode_without_workspace(decode_data, m):
    import oracle as orc
    weights, xs = decode_data
    qw, sfw, gw, gsfw = weights["qkv"]
    n, k = synthetic.DECODE_SHAPES["qkv"]
    x = xs[k][:m].contiguous()
    qx, sfx = orc.mx_quantize(synthetic.bits(x))
    gx, gsfx = fp8mm.mxfp8_quantize(gu.to_dev(x))
    c = fp8mm.mxfp8_gemm(gx, gsfx, gw, gsfw)
    torch.cuda.synchronize()
    c_ref, bound = orc.gemm_mx(qx, sfx, qw, sfw)
    gu.check_gemm(c, c_ref, bound, f"decode qkv m={m} one CTA per tile")


@pytest.mark.parametrize("ctas", [1, 7, 37, 300, 5000])
def test_decode_partitions(decode_data, ctas):
    """Different stream-K partitions (including more CTAs than units) all meet
    the bar; each partition is deterministic."""
    import oracle as orc
    weights, xs = decode_data
    qw, sfw, gw, gsfw = weights["down"]
    n, k = synthetic.DECODE_SHAPES["down"]
    m = 8
    x = xs[k][:m].contiguous()
    qx, sfx = orc.mx_quantize(synthetic.bits(x))
    gx, gsfx = fp8mm.mxfp8_quantize(gu.to_dev(x))
    ws = _workspace(m, n, k, ctas)
    c1 = fp8mm.mxfp8_gemm(gx, gsfx, gw, gsfw, workspace=ws, small_m_ctas=ctas)
    c2 = fp8mm.mxfp8_gemm(gx, gsfx, gw, gsfw, workspace=ws, small_m_ctas=ctas)
    torch.cuda.synchronize()
    c_ref, bound = orc.gemm_mx(qx, sfx, qw, sfw)
    gu.check_gemm(c1, c_ref, bound, f"decode down m=8 ctas={ctas}")
    assert torch.equal(c1, c2)


@pytest.mark.parametrize("name,m,ctas", [("down", 8, 96), ("down", 33, 288), ("qkv", 8, 144), ("qkv", 64, 240)])
def test_decode_multiple_of_tiles_partitions(decode_data, name, m, ctas):
    """CTA counts that are multiples of the tile count whose quotient does not
    divide the tile's K slabs (112 / 3, 112 / 9, 32 / 3, 32 / 5), so ranges
    cross tiles at shifting offsets; with 33 tokens and 64 tokens (48- and
    64-token tiles, one CTA per SM, so more CTAs than fit at once)."""
    import oracle as orc
    weights, xs = decode_data
    qw, sfw, gw, gsfw = weights[name]
    n, k = synthetic.DECODE_SHAPES[name]
    x = xs[k][:m].contiguous()
    qx, sfx = orc.mx_quantize(synthetic.bits(x))
    gx, gsfx = fp8mm.mxfp8_quantize(gu.to_dev(x))
    ws = _workspace(m, n, k, ctas)
    c1 = fp8mm.mxfp8_gemm(gx, gsfx, gw, gsfw, workspace=ws, small_m_ctas=ctas)
    c2 = fp8mm.mxfp8_gemm(gx, gsfx, gw, gsfw, workspace=ws, small_m_ctas=ctas)
    torch.cuda.synchronize()
    c_ref, bound = orc.gemm_mx(qx, sfx, qw, sfw)
    gu.check_gemm(c1, c_ref, bound, f"decode {name} m={m} ctas={ctas}")
    assert torch.equal(c1, c2)


@pytest.mark.parametrize("m,n,k", [(3, 200, 96), (17, 130, 4128), (64, 384, 320), (33, 1000, 64)])
def test_decode_ragged(m, n, k):
    """Ragged shapes; the weights are quantized right before each GEMM on the
    same stream, so the GEMM must not read them before that kernel ends
    (no weights_ready flag)."""
    import oracle as orc
    x = synthetic.random_bf16((m, k), seed=m * 3 + k)
    w = synthetic.random_bf16((n, k), seed=n * 5 + k, sigma=0.02)
    qx, sfx = orc.mx_quantize(synthetic.bits(x))
    qw, sfw = orc.mx_quantize(synthetic.bits(w))
    gx, gsfx = fp8mm.mxfp8_quantize(gu.to_dev(x))
    gw, gsfw = fp8mm.mxfp8_quantize(gu.to_dev(w))
    c_ref, bound = orc.gemm_mx(qx, sfx, qw, sfw)
    for ctas in (0, 5, 10, 66):                                  # 2 tiles x 33 slabs at k = 4128
        ws = _workspace(m, n, k, ctas)
        gw, gsfw = fp8mm.mxfp8_quantize(gu.to_dev(w))          # immediately precedes the GEMM
        c = fp8mm.mxfp8_gemm(gx, gsfx, gw, gsfw, workspace=ws, small_m_ctas=ctas)
        torch.cuda.synchronize()
        gu.check_gemm(c, c_ref, bound, f"decode ragged {m}x{n}x{k} ctas={ctas}")
    c = fp8mm.mxfp8_gemm(gx, gsfx, gw, gsfw, kernel=fp8mm.KERNEL_TILED)
    torch.cuda.synchronize()
    gu.check_gemm(c, c_ref, bound, f"tiled {m}x{n}x{k}")


def test_workspace_too_small_is_rejected(decode_data):
    weights, xs = decode_data
    _, _, gw, gsfw = weights["qkv"]
    n, k = synthetic.DECODE_SHAPES["qkv"]
    gx, gsfx = fp8mm.mxfp8_quantize(gu.to_dev(xs[k][:8].contiguous()))
    ws = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(fp8mm.Fp8mmError):                       # a split reduced through the workspace
        fp8mm.mxfp8_gemm(gx, gsfx, gw, gsfw, workspace=ws, split_via_workspace=True)
    with pytest.raises(fp8mm.Fp8mmError):                       # 37 CTAs: not tile-aligned
        fp8mm.mxfp8_gemm(gx, gsfx, gw, gsfw, workspace=ws, small_m_ctas=37)


# ------------------------------------------------------------ tile-aligned splits reduced in clusters

N_TILES = {name: -(-n // 128) for name, (n, k) in synthetic.DECODE_SHAPES.items()}


@pytest.mark.parametrize("name,m,s", [("qkv", 1, 4), ("qkv", 64, 2), ("up", 8, 2), ("up", 32, 4), ("up", 64, 8),
                                      ("down", 1, 8), ("down", 16, 7), ("down", 48, 4), ("down", 64, 2),
                                      ("qkv", 1, 3), ("qkv", 16, 5), ("qkv", 64, 6), ("up", 1, 3),
                                      ("down", 8, 3), ("down", 32, 5), ("down", 64, 6)])
def test_cluster_reduction_equals_workspace_reduction(decode_data, name, m, s):
    """s CTAs per weight tile (2 <= s <= 8; the tile's K slabs -- 32 for up
    and qkv, 112 for down -- split as floor(r*num_k/s), so s need not divide
    them) are reduced inside a cluster through distributed shared memory; the
    same partition reduced through the workspace gives identical bits, and
    both meet the bar."""
    import oracle as orc
    weights, xs = decode_data
    qw, sfw, gw, gsfw = weights[name]
    n, k = synthetic.DECODE_SHAPES[name]
    ctas = N_TILES[name] * s
    x = xs[k][:m].contiguous()
    qx, sfx = orc.mx_quantize(synthetic.bits(x))
    gx, gsfx = fp8mm.mxfp8_quantize(gu.to_dev(x))
    ws = _workspace(m, n, k, ctas)
    c_cl = fp8mm.mxfp8_gemm(gx, gsfx, gw, gsfw, small_m_ctas=ctas, weights_ready=True)   # no workspace needed
    c_cl2 = fp8mm.mxfp8_gemm(gx, gsfx, gw, gsfw, workspace=ws, small_m_ctas=ctas)
    torch.cuda.synchronize()
    assert not ws.any()                                          # the cluster path leaves a workspace alone
    c_ws = fp8mm.mxfp8_gemm(gx, gsfx, gw, gsfw, workspace=ws, small_m_ctas=ctas, split_via_workspace=True)
    torch.cuda.synchronize()
    c_ref, bound = orc.gemm_mx(qx, sfx, qw, sfw)
    gu.check_gemm(c_cl, c_ref, bound, f"cluster reduction {name} m={m} s={s}")
    assert torch.equal(c_cl, c_ws) and torch.equal(c_cl, c_cl2)
    tickets = -(-N_TILES[name] * 4 // 256) * 256
    assert not ws[-tickets:].any()                               # the workspace path reset its counters
    assert fp8mm.last_device_error() == 0


@pytest.mark.parametrize("m,n,k,s", [(5, 200, 512, 2), (17, 130, 4096, 8), (40, 384, 896, 7), (64, 257, 1024, 4),
                                     (9, 300, 896, 5), (33, 140, 640, 3), (2, 129, 768, 6)])
def test_cluster_reduction_ragged(m, n, k, s):
    """Ragged weight tiles (n not a multiple of 128) and token counts that fill
    part of the 16/32/48/64-token tile, with 2..8 CTAs per tile, some of which
    do not divide the tile's K slabs (7 slabs in 5 parts, 5 in 3, 6 in 6)."""
    import oracle as orc
    x = synthetic.random_bf16((m, k), seed=m * 7 + k)
    w = synthetic.random_bf16((n, k), seed=n * 11 + k, sigma=0.02)
    qx, sfx = orc.mx_quantize(synthetic.bits(x))
    qw, sfw = orc.mx_quantize(synthetic.bits(w))
    gx, gsfx = fp8mm.mxfp8_quantize(gu.to_dev(x))
    gw, gsfw = fp8mm.mxfp8_quantize(gu.to_dev(w))
    ctas = -(-n // 128) * s
    c = fp8mm.mxfp8_gemm(gx, gsfx, gw, gsfw, small_m_ctas=ctas)
    ws = _workspace(m, n, k, ctas)
    c_ws = fp8mm.mxfp8_gemm(gx, gsfx, gw, gsfw, workspace=ws, small_m_ctas=ctas, split_via_workspace=True)
    torch.cuda.synchronize()
    c_ref, bound = orc.gemm_mx(qx, sfx, qw, sfw)
    gu.check_gemm(c, c_ref, bound, f"cluster reduction ragged {m}x{n}x{k} s={s}")
    assert torch.equal(c, c_ws)
    assert fp8mm.last_device_error() == 0
