"""Per-tensor scale, static-scale quantizer and the E4M3-output GEMM against
the CPU oracle (page "FP8 推理基础设施（五）：从 DeepGEMM 到 vLLM", listing 3:
one scale max|x| / 448 per tensor; listing 1: the GEMM's C_fp8 output).
Scales and codes must match bit for bit.  The E4M3 GEMM output cannot be
unique (the fp32 tensor-core sum is within the GEMM tolerance of the exact
one), so each code must lie between the codes of the ends of the tolerance
interval around the exact result divided by the output scale."""
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


def _scale_both(x_cpu):
    import oracle as orc
    s_ref = orc.tensor_scale(synthetic.bits(x_cpu))
    s = fp8mm.fp8_tensor_scale(gu.to_dev(x_cpu))
    torch.cuda.synchronize()
    return float(s.item()), float(s_ref)


def _static_both(x_cpu, scale: float):
    import oracle as orc
    q_ref = orc.quantize_static(synthetic.bits(x_cpu), np.float32(scale))
    s = torch.tensor([scale], dtype=torch.float32, device="cuda")
    q = fp8mm.fp8_quantize_static(gu.to_dev(x_cpu), s)
    torch.cuda.synchronize()
    return q.cpu().numpy(), q_ref


def test_tensor_scale_matches_the_oracle():
    a, _ = synthetic.attn()
    cases = [a, synthetic.random_bf16((300, 480), seed=3, sigma=7.0), synthetic.random_bf16((5, 8), seed=4)]
    cases[1][17, 33] = 1e4
    tiny = synthetic.random_bf16((64, 64), seed=5) * 1e-38
    cases += [tiny, torch.zeros((16, 32), dtype=torch.bfloat16)]
    for x in cases:
        s, s_ref = _scale_both(x)
        assert np.float32(s).view(np.uint32) == np.float32(s_ref).view(np.uint32), (x.shape, s, s_ref)
    s = fp8mm.fp8_tensor_scale(torch.empty((0, 64), dtype=torch.bfloat16, device="cuda"))
    assert s.item() == 1.0


def test_tensor_scale_strided_and_repeated():
    """A strided view (row stride 200, k 128: values past the view must not
    count), rows spread over many blocks, and repeated calls on one output
    word (each call starts from its own zeroed word)."""
    import oracle as orc
    base = synthetic.random_bf16((1000, 200), seed=8, sigma=3.0)
    base[999, 100] = 5e3                                   # inside the view: the maximum
    base[500, 190] = 1e6                                   # outside the view
    view_d = gu.to_dev(base)[:, :128]
    s_ref = orc.tensor_scale(synthetic.bits(base[:, :128].contiguous()))
    out = torch.empty(1, dtype=torch.float32, device="cuda")
    for _ in range(3):
        fp8mm.fp8_tensor_scale(view_d, out)
        torch.cuda.synchronize()
        assert np.float32(out.item()).view(np.uint32) == np.float32(s_ref).view(np.uint32)
    big = synthetic.random_bf16((4096, 4096), seed=9)
    big[4095, 4095] = -300.0
    s, s_ref = _scale_both(big)
    assert np.float32(s).view(np.uint32) == np.float32(s_ref).view(np.uint32)


@pytest.mark.parametrize("scale", [1.0, 0.0078125, 3.0e-3, 1.7, 12345.0, 2.0 ** -85, 2.0 ** 127, 1.0e-30])
def test_static_quantizer_every_bf16_value(scale):
    """All finite bf16 values at scales that keep the quotient in range, push
    most of it past 448 (saturation) or below the E4M3 subnormals, and scales
    outside [2^-80, 2^126] where the kernel divides."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    v = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
    v = v[torch.isfinite(v.float())]
    n = v.numel() // 64 * 64
    x = v[:n].reshape(-1, 64).contiguous()
    q, q_ref = _static_both(x, scale)
    bad = np.argwhere(q != q_ref)
    assert bad.size == 0, f"scale {scale}: {len(bad)} mismatches, first {bad[:4].tolist()}"


def test_static_with_the_tensor_scale_on_workloads():
    a, _ = synthetic.attn()
    for x in (a, synthetic.random_bf16((129, 4096), seed=7, sigma=0.05)):
        s, _ = _scale_both(x)
        q, q_ref = _static_both(x, s)
        assert np.array_equal(q, q_ref)


def test_static_strided_and_ragged():
    import oracle as orc
    base = synthetic.random_bf16((33, 200), seed=8)
    view = base[:, :152]
    s = torch.tensor([0.02], dtype=torch.float32, device="cuda")
    q = torch.zeros((33, 160), dtype=torch.uint8, device="cuda")
    fp8mm.fp8_quantize_static(gu.to_dev(base)[:, :152], s, q[:, :152])
    torch.cuda.synchronize()
    q_ref = orc.quantize_static(synthetic.bits(view.contiguous()), np.float32(0.02))
    assert np.array_equal(q[:, :152].cpu().numpy(), q_ref)
    assert not q[:, 152:].any()                                  # nothing past k is written


def _check_e4m3_gemm(c_codes, c_ref, bound, s_out, label):
    import oracle as orc
    dec = orc.e4m3_decode_table()
    tol = gu.ABS_BOUND_FACTOR * bound + gu.REL_FACTOR * np.abs(c_ref)
    lo = orc.e4m3_encode(((c_ref - tol) / s_out).ravel())
    hi = orc.e4m3_encode(((c_ref + tol) / s_out).ravel())
    got = dec[c_codes.ravel()]
    ok = (got >= dec[lo]) & (got <= dec[hi])
    bad = np.nonzero(~ok)[0]
    assert bad.size == 0, (f"{label}: {bad.size} codes outside the tolerance interval, first at {bad[:3]}: "
                           f"got {got[bad[:3]]}, interval [{dec[lo][bad[:3]]}, {dec[hi][bad[:3]]}]")


@pytest.mark.parametrize("kernel", [fp8mm.KERNEL_AUTO, fp8mm.KERNEL_TILED_1SM, fp8mm.KERNEL_TILED_2SM,
                                    fp8mm.KERNEL_TILED_1SM_N128])
def test_e4m3_out_tiny_and_ragged(kernel):
    import oracle as orc
    for (m, n, k) in [(128, 256, 512), (300, 130, 96), (257, 513, 1040)]:
        a = synthetic.random_bf16((m, k), seed=m + k)
        bt = synthetic.random_bf16((n, k), seed=n + 2 * k)
        qa, sa = orc.quantize_rowwise(synthetic.bits(a))
        qb, sb = orc.quantize_rowwise(synthetic.bits(bt))
        c_ref, bound = orc.gemm_rowwise(qa, qb, sa, sb)
        s_out = np.float32(np.abs(c_ref).max() / 448.0 * 0.7)    # 30 % of the outputs saturate-free headroom
        ga, gsa = fp8mm.fp8_quantize_rowwise(gu.to_dev(a))
        gb, gsb = fp8mm.fp8_quantize_rowwise(gu.to_dev(bt))
        so = torch.tensor([s_out], dtype=torch.float32, device="cuda")
        c = fp8mm.fp8_gemm_e4m3_out(ga, gb, gsa, gsb, so, kernel=kernel)
        torch.cuda.synchronize()
        _check_e4m3_gemm(c.cpu().numpy(), c_ref, bound, s_out, f"{m}x{n}x{k} kernel {kernel}")


def test_e4m3_out_attn_sampled_and_strided():
    import oracle as orc
    a, bt = synthetic.attn()
    ga, gsa = fp8mm.fp8_quantize_rowwise(gu.to_dev(a))
    gb, gsb = fp8mm.fp8_quantize_rowwise(gu.to_dev(bt))
    so = torch.tensor([0.5], dtype=torch.float32, device="cuda")
    c = torch.zeros((8192, 2048 + 16), dtype=torch.uint8, device="cuda")[:, :2048]
    fp8mm.fp8_gemm_e4m3_out(ga, gb, gsa, gsb, so, c=c)
    torch.cuda.synchronize()
    qa, sa = ga.cpu().numpy(), gsa.cpu().numpy()
    qb, sb = gb.cpu().numpy(), gsb.cpu().numpy()
    rows = np.random.default_rng(11).choice(8192, 48, replace=False)
    c_ref, bound = orc.gemm_rowwise(qa[rows], qb, sa[rows], sb)
    _check_e4m3_gemm(c[torch.from_numpy(rows).cuda()].cpu().numpy(), c_ref, bound, 0.5, "attn e4m3 out")


def test_e4m3_out_bf16_agreement_and_errors():
    """Where the bf16 and E4M3 outputs come from the same accumulator, the
    E4M3 code is the encoding of a value within one bf16 rounding of the bf16
    output; and bad arguments are rejected."""
    a = synthetic.random_bf16((256, 512), seed=21)
    bt = synthetic.random_bf16((384, 512), seed=22)
    ga, gsa = fp8mm.fp8_quantize_rowwise(gu.to_dev(a))
    gb, gsb = fp8mm.fp8_quantize_rowwise(gu.to_dev(bt))
    so = torch.tensor([1.0], dtype=torch.float32, device="cuda")
    c8 = fp8mm.fp8_gemm_e4m3_out(ga, gb, gsa, gsb, so)
    cb = fp8mm.fp8_gemm(ga, gb, gsa, gsb)
    torch.cuda.synchronize()
    import oracle as orc
    dec = orc.e4m3_decode_table()
    v = cb.float().cpu().numpy().astype(np.float64)
    lo = orc.e4m3_encode((v - np.abs(v) * 2.0 ** -8).ravel())
    hi = orc.e4m3_encode((v + np.abs(v) * 2.0 ** -8).ravel())
    got = dec[c8.cpu().numpy().ravel()]
    assert np.all((got >= dec[lo]) & (got <= dec[hi]))
    with pytest.raises(fp8mm.Fp8mmError):
        fp8mm.fp8_gemm_e4m3_out(ga, gb, gsa, gsb, so, kernel=fp8mm.KERNEL_SMALL_M)
    bad = torch.zeros((256, 500), dtype=torch.uint8, device="cuda")
    with pytest.raises(fp8mm.Fp8mmError):
        fp8mm.fp8_gemm_e4m3_out(bad, gb[:, :500].contiguous(), gsa, gsb, so)   # k % 16 != 0
    assert fp8mm.last_device_error() == 0
