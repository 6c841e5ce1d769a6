"""Every kernel launched with programmatic dependent launch (the quantizers,
the per-tensor kernels, the MLA key assembly, the small-M and tiled GEMMs)
may start while the preceding kernel on the stream is still running and must
read its inputs, and write its outputs, only after that kernel is done.  Each case rewrites the input with a
torch kernel immediately before the call, several times with different
values, and compares with the same call on a fresh, fully written copy."""
import pytest
import torch

import mxfp8_block_scaled_fp8_b200 as fp8mm
from mxfp8_block_scaled_fp8_b200 import synthetic
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    gu.require_gpu()


SCALES = (1.0, -3.0, 0.25, 7.5)


def _rewrite_then(op, x0, buf):
    """op(buf) right after torch writes buf = x0 * scale, vs op on a separate copy."""
    for scale in SCALES:
        torch.mul(x0, scale, out=buf)          # the preceding kernel on the stream
        got = op(buf)
        ref_in = (x0 * scale).contiguous()
        torch.cuda.synchronize()
        ref = op(ref_in)
        torch.cuda.synchronize()
        for g, r in zip(got if isinstance(got, tuple) else (got,), ref if isinstance(ref, tuple) else (ref,)):
            assert torch.equal(g, r), f"scale {scale}"


def test_quantizers_read_after_the_preceding_kernel():
    x0 = gu.to_dev(synthetic.random_bf16((512, 4096), seed=41))
    buf = torch.empty_like(x0)
    _rewrite_then(lambda x: tuple(t.clone() for t in fp8mm.fp8_quantize_rowwise(x)), x0, buf)
    _rewrite_then(lambda x: tuple(t.clone() for t in fp8mm.mxfp8_quantize(x)), x0, buf)
    _rewrite_then(lambda x: fp8mm.fp8_tensor_scale(x).clone(), x0, buf)
    s = torch.tensor([0.01], dtype=torch.float32, device="cuda")
    _rewrite_then(lambda x: fp8mm.fp8_quantize_static(x, s).clone(), x0, buf)


def test_static_quantizer_reads_the_scale_after_the_preceding_kernel():
    x = gu.to_dev(synthetic.random_bf16((256, 1024), seed=42))
    for v in (0.5, 0.003, 11.0):
        s = torch.empty(1, dtype=torch.float32, device="cuda")
        s.fill_(v)                              # written by the kernel right before
        q = fp8mm.fp8_quantize_static(x, s)
        ref = fp8mm.fp8_quantize_static(x, torch.tensor([v], dtype=torch.float32, device="cuda"))
        torch.cuda.synchronize()
        assert torch.equal(q, ref)


def test_concat_reads_after_the_preceding_kernel():
    g = torch.Generator(device="cuda").manual_seed(43)
    nope0 = torch.randint(0, 120, (64, 16, 128), device="cuda", dtype=torch.uint8, generator=g)
    rope = torch.randint(0, 120, (64, 1, 64), device="cuda", dtype=torch.uint8, generator=g)
    buf = torch.empty_like(nope0)
    for add in (1, 2, 3):
        torch.add(nope0, add, out=buf)
        got = fp8mm.concat_mla_k(buf, rope)
        torch.cuda.synchronize()
        ref = torch.cat([nope0 + add, rope.expand(64, 16, 64)], dim=2)
        assert torch.equal(got, ref)


def test_small_m_gemm_reads_the_activation_after_the_preceding_kernel():
    w = gu.to_dev(synthetic.random_bf16((1024, 2048), seed=44, sigma=0.02))
    qw, sfw = fp8mm.mxfp8_quantize(w)
    x0 = gu.to_dev(synthetic.random_bf16((8, 2048), seed=45))
    qx0, sfx0 = fp8mm.mxfp8_quantize(x0)
    ws = torch.zeros(fp8mm.workspace_bytes(8, 1024, 2048), dtype=torch.uint8, device="cuda")
    qx = torch.empty_like(qx0)
    for v in (0, 1, 2):
        qx.copy_(qx0 if v == 0 else torch.flip(qx0, dims=[v - 1]))   # written right before the GEMM
        c = fp8mm.mxfp8_gemm(qx, sfx0, qw, sfw, workspace=ws, weights_ready=True)
        ref = fp8mm.mxfp8_gemm(qx.clone(), sfx0, qw, sfw, workspace=ws, weights_ready=True)
        torch.cuda.synchronize()
        assert torch.equal(c, ref)


TILED = [fp8mm.KERNEL_TILED_2SM, fp8mm.KERNEL_TILED_1SM, fp8mm.KERNEL_TILED_1SM_N128]


@pytest.mark.parametrize("kernel", TILED, ids=["2sm", "1sm", "1sm_n128"])
def test_tiled_gemms_read_after_the_preceding_kernel(kernel):
    """The tiled GEMMs (also launched with programmatic dependent launch) see A, its scales and the per-token
    scales as the kernel right before them wrote them."""
    a0 = gu.to_dev(synthetic.random_bf16((512, 1024), seed=46))
    b = gu.to_dev(synthetic.random_bf16((768, 1024), seed=47, sigma=0.05))
    qa0, sfa0 = fp8mm.mxfp8_quantize(a0)
    qb, sfb = fp8mm.mxfp8_quantize(b)
    qa = torch.empty_like(qa0)
    for v in (0, 1, 2):
        qa.copy_(qa0 if v == 0 else torch.flip(qa0, dims=[v - 1]))   # written right before the GEMM
        c = fp8mm.mxfp8_gemm(qa, sfa0, qb, sfb, kernel=kernel)
        ref = fp8mm.mxfp8_gemm(qa.clone(), sfa0, qb, sfb, kernel=kernel)
        torch.cuda.synchronize()
        assert torch.equal(c, ref)
    ra0, sa0 = fp8mm.fp8_quantize_rowwise(a0)
    rb, sb = fp8mm.fp8_quantize_rowwise(b)
    sa = torch.empty_like(sa0)
    for scale in (1.0, 0.5, 3.0):
        torch.mul(sa0, scale, out=sa)                                # written right before the GEMM
        c = fp8mm.fp8_gemm(ra0, rb, sa, sb, kernel=kernel)
        ref = fp8mm.fp8_gemm(ra0, rb, (sa0 * scale).contiguous(), sb, kernel=kernel)
        torch.cuda.synchronize()
        assert torch.equal(c, ref)


@pytest.mark.parametrize("kernel", TILED, ids=["2sm", "1sm", "1sm_n128"])
def test_tiled_gemm_writes_c_after_the_preceding_kernel_read_it(kernel):
    """C of a tiled GEMM is the input of the quantizer right before it on the stream: the quantizer's codes
    are those of the old contents (the GEMM's epilogue waits for the quantizer before its first store)."""
    m, n, k = 512, 2048, 1024
    a = gu.to_dev(synthetic.random_bf16((m, k), seed=48))
    b = gu.to_dev(synthetic.random_bf16((n, k), seed=49, sigma=0.05))
    qa, sfa = fp8mm.mxfp8_quantize(a)
    qb, sfb = fp8mm.mxfp8_quantize(b)
    for seed in (50, 51):
        x = gu.to_dev(synthetic.random_bf16((m, n), seed=seed))
        ref_q, ref_sf = (t.clone() for t in fp8mm.mxfp8_quantize(x.clone()))
        q, sf = fp8mm.mxfp8_quantize(x)                              # reads x ...
        fp8mm.mxfp8_gemm(qa, sfa, qb, sfb, c=x, kernel=kernel)      # ... which the GEMM then overwrites
        torch.cuda.synchronize()
        assert torch.equal(q, ref_q) and torch.equal(sf, ref_sf)
        assert torch.equal(x, fp8mm.mxfp8_gemm(qa, sfa, qb, sfb, kernel=kernel))
