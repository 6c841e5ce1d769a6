"""GPU quantizers vs the CPU oracle: codes, scales and scale-layout bytes must
match bit for bit (page "从 DeepGEMM 到 vLLM", listing 3 rule per row; page
"[sglang] FlashInfer v0.6.7 MXFP8 Gemm 통합", section 1, one UE8M0 scale per
32 elements)."""
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


def _rowwise_both(orc, x_cpu: torch.Tensor):
    q_ref, s_ref = orc.quantize_rowwise(synthetic.bits(x_cpu))
    q, s = fp8mm.fp8_quantize_rowwise(gu.to_dev(x_cpu))
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy(), q_ref, s_ref


def _assert_rowwise(orc, x_cpu, label):
    q, s, q_ref, s_ref = _rowwise_both(orc, x_cpu)
    bad_s = np.nonzero(s.view(np.uint32) != s_ref.view(np.uint32))[0]
    assert bad_s.size == 0, f"{label}: scale mismatch at rows {bad_s[:8]}: {s[bad_s[:4]]} vs {s_ref[bad_s[:4]]}"
    bad = np.argwhere(q != q_ref)
    assert bad.size == 0, f"{label}: {len(bad)} code mismatches, first {bad[:4].tolist()}"


def _assert_mx(orc, x_cpu, label):
    rows, k = x_cpu.shape
    q_ref, sf_ref = orc.mx_quantize(synthetic.bits(x_cpu))
    q, sf = fp8mm.mxfp8_quantize(gu.to_dev(x_cpu))
    torch.cuda.synchronize()
    q = q.cpu().numpy()
    sf = sf.cpu().numpy()
    bad = np.argwhere(q != q_ref)
    assert bad.size == 0, f"{label}: {len(bad)} code mismatches, first {bad[:4].tolist()}"
    canon = gu.sf_canonical_from_layout(sf, rows, k)
    bad = np.argwhere(canon != sf_ref)
    assert bad.size == 0, f"{label}: {len(bad)} scale mismatches, first {bad[:4].tolist()}"
    # the whole buffer: real bytes where the layout says, zero padding elsewhere
    assert np.array_equal(sf, gu.sf_layout_from_canonical(sf_ref, rows, k)), f"{label}: padding bytes"
    # the library's own permutation helper agrees with the formula
    assert np.array_equal(fp8mm.sf_to_canonical(torch.from_numpy(sf), rows, k).numpy(), sf_ref)


# ------------------------------------------------------------ workloads

def test_rowwise_tiny():
    import oracle as orc
    a, bt = synthetic.tiny()
    _assert_rowwise(orc, a, "tiny A")
    _assert_rowwise(orc, bt, "tiny B^T")


def test_rowwise_attn_full_size():
    import oracle as orc
    a, bt = synthetic.attn()
    _assert_rowwise(orc, a, "attn A 8192x8192")
    _assert_rowwise(orc, bt, "attn B^T 2048x8192")


def test_mx_qk_full_size():
    import oracle as orc
    a, bt = synthetic.qk()
    _assert_mx(orc, a, "qk A 2048x4096 (outlier rows)")
    _assert_mx(orc, bt, "qk B^T 1024x4096 (outlier cols)")


def test_mx_ffn_up_full_size():
    import oracle as orc
    x, w = synthetic.ffn_up()
    _assert_mx(orc, x, "ffn_up X 8192x8192")
    _assert_mx(orc, w, "ffn_up W 22016x8192 (0.1% x20 outliers)")


def test_mx_decode_shapes():
    import oracle as orc
    ws, xs = synthetic.decode()
    for name, w in ws.items():
        _assert_mx(orc, w, f"decode W {name} {tuple(w.shape)}")
    for k, x in xs.items():
        for m in synthetic.DECODE_M:
            _assert_mx(orc, x[:m].contiguous(), f"decode X m={m} k={k}")


def test_quantizers_on_the_other_mode_shapes():
    """Both quantizers on every configuration's activation shape."""
    import oracle as orc
    a, _ = synthetic.qk()
    _assert_rowwise(orc, a, "qk A rowwise")
    a, _ = synthetic.tiny()
    _assert_mx(orc, a, "tiny A mx")


# ------------------------------------------------------------ edge cases

def _edge_tensor():
    x = synthetic.random_bf16((300, 480), seed=21, sigma=2.0)
    x[0] = 0.0                                          # all-zero row
    x[1] = -0.0
    x[2, :] = 3.0                                       # constant row
    x[3] *= 1e-38                                       # bf16 subnormals
    x[4] = torch.finfo(torch.bfloat16).max              # max magnitude
    x[4, 1::2] = -torch.finfo(torch.bfloat16).max
    x[5, :32] = 0.0                                     # a zero block inside a row
    x[6, 32:64] = 448.0 * 2 ** -9                       # amax exactly 448 * 2^j
    x[7] *= 1e30
    return x


@pytest.mark.parametrize("rows,k", [(1, 512), (200, 96), (129, 4096), (3, 32), (64, 14336),
                                    # few rows and a long K: the one-warp-per-scale-line kernel
                                    (1, 8192), (17, 8224), (32, 14336), (5, 9984)])
def test_mx_ragged_and_small(rows, k):
    import oracle as orc
    _assert_mx(orc, synthetic.random_bf16((rows, k), seed=rows + k), f"mx {rows}x{k}")


@pytest.mark.parametrize("rows,k", [(1, 512), (200, 40), (129, 4096), (3, 8), (5, 20000), (64, 14336)])
def test_rowwise_ragged_and_small(rows, k):
    import oracle as orc
    _assert_rowwise(orc, synthetic.random_bf16((rows, k), seed=rows * 7 + k), f"rowwise {rows}x{k}")


def test_edge_values_both_modes():
    import oracle as orc
    x = _edge_tensor()
    _assert_rowwise(orc, x, "edge rowwise")
    _assert_mx(orc, x, "edge mx")


def test_every_bf16_value_converts_like_the_oracle():
    """All finite bf16 values with |x| <= 448, laid out so every 32-block's
    maximum is 448 (MX scale 2^0) and every row's maximum is 448 (scale 1):
    the E4M3 conversion itself is compared exhaustively, midpoints included."""
    import oracle as orc
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
    f = vals.float()
    keep = torch.isfinite(f) & (f.abs() <= 448.0)
    vals = vals[keep]
    n = vals.numel()
    per = 31                                            # 31 values + one 448 per block
    nblk = -(-n // per)
    flat = torch.zeros(nblk * per, dtype=torch.bfloat16)
    flat[:n] = vals
    blocks = torch.zeros((nblk, 32), dtype=torch.bfloat16)
    blocks[:, 0] = 448.0
    blocks[:, 1:] = flat.view(nblk, per)
    rows = -(-nblk // 16)                               # 16 blocks (512 elements) per row
    padded = torch.zeros((rows * 16, 32), dtype=torch.bfloat16)
    padded[:nblk] = blocks
    padded[nblk:, 0] = 448.0
    x2 = padded.view(rows, 16 * 32).contiguous()
    _assert_mx(orc, x2, "all bf16 values, mx scale 1")
    _assert_rowwise(orc, x2, "all bf16 values, rowwise scale 1")


def test_rowwise_many_scales_and_magnitudes():
    """Per-row quotients x / s over many scales: each row's maximum is a random
    bf16 over 2^-40..2^40 with a random mantissa, its other values spread
    log-uniformly over 40 binades below it, so quotients fall in every E4M3
    binade, the subnormal codes and below, and some lie next to rounding
    midpoints; rows with subnormal or huge maxima are included."""
    import oracle as orc
    g = np.random.default_rng(77)
    rows, k = 2048, 1024
    amax = np.ldexp(1.0 + g.random(rows), g.integers(-40, 41, rows))
    amax[:4] = [1e-39, 3e-36, 2.0 ** 126, 3.0e38]                # 1/s overflows; subnormal s; huge
    mag = np.exp2(-40.0 * g.random((rows, k))) * amax[:, None]
    x = np.where(g.random((rows, k)) < 0.5, -mag, mag)
    x[np.arange(rows), g.integers(0, k, rows)] = amax           # the row maximum itself
    xt = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    _assert_rowwise(orc, xt, "rowwise many scales")


def test_strided_input_rows():
    import oracle as orc
    base = synthetic.random_bf16((50, 640), seed=5)
    view = base[:, :512]                                # row stride 640 elements
    q_ref, s_ref = orc.quantize_rowwise(synthetic.bits(view.contiguous()))
    q, s = fp8mm.fp8_quantize_rowwise(gu.to_dev(base)[:, :512])
    assert np.array_equal(q.cpu().numpy(), q_ref) and np.array_equal(s.cpu().numpy(), s_ref)
    q_ref, sf_ref = orc.mx_quantize(synthetic.bits(view.contiguous()))
    q, sf = fp8mm.mxfp8_quantize(gu.to_dev(base)[:, :512])
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(gu.sf_canonical_from_layout(sf.cpu().numpy(), 50, 512), sf_ref)


def test_empty_inputs():
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    q, s = fp8mm.fp8_quantize_rowwise(x)
    q, sf = fp8mm.mxfp8_quantize(x)
    x = torch.empty((4, 0), dtype=torch.bfloat16, device="cuda")
    q, s = fp8mm.fp8_quantize_rowwise(x)
    torch.cuda.synchronize()
    assert torch.all(s == 1.0)


def test_bad_arguments_are_rejected():
    x = torch.zeros((4, 40), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fp8mm.Fp8mmError):
        fp8mm.mxfp8_quantize(x)                         # k % 32 != 0
    x = torch.zeros((4, 12), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fp8mm.Fp8mmError):
        fp8mm.fp8_quantize_rowwise(x)                   # k % 8 != 0


def test_mx_few_rows_long_k_strided_and_unaligned_q():
    """The one-warp-per-scale-line kernel (few rows, long K) on a strided
    input and an output whose rows are only 8-byte aligned."""
    import oracle as orc
    base = synthetic.random_bf16((20, 8704), seed=15, sigma=4.0)
    base[3, 100:200] = 0.0
    view = base[:, :8192]
    q_ref, sf_ref = orc.mx_quantize(synthetic.bits(view.contiguous()))
    qbuf = torch.zeros((20, 8200), dtype=torch.uint8, device="cuda")   # row stride 8200: 8-byte aligned rows
    q, sf = fp8mm.mxfp8_quantize(gu.to_dev(base)[:, :8192], q=qbuf[:, :8192])
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(sf.cpu().numpy(), gu.sf_layout_from_canonical(sf_ref, 20, 8192))
