"""Pins for the fp32 quotient step of the oracle's two scale-based quantizers.

Both `orc_quantize_rowwise` and `orc_quantize_static` form fp32(x / s) and then
round that to E4M3: the scale rule is max|x| / 448 (page "FP8 推理基础设施（五）：
从 DeepGEMM 到 vLLM", listing 3) and the reading taken where the pages are silent
is an IEEE (correctly rounded) fp32 quotient followed by a round-to-nearest-even,
saturating E4M3 conversion.  The independent reference here is torch's own CPU
arithmetic: an fp32 tensor division and torch's float8_e4m3fn cast after
clamping to +-448.

The inputs are chosen so that a reciprocal-multiply quotient, fp32(x * fp32(1/s)),
lands on the other side of an E4M3 rounding midpoint for some elements: rows
whose maximum a has any of the 128 bf16 significands and elements x with x / s
at a tie (e.g. a = 1.078125, x = 0.75 a: x / s = 336, midway between the codes
320 and 352).  Each test checks that its input really has such elements, so a
planted `x * (1.0f / s)` cannot pass."""
import numpy as np
import torch

from mxfp8_block_scaled_fp8_b200 import synthetic

DIVISOR = 448.0   # the scale rule's divisor (E4M3 max finite)


def _codes(q: torch.Tensor) -> np.ndarray:
    return q.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _torch_rowwise(x: torch.Tensor):
    """torch's fp32 arithmetic: s = amax / 448 per row (1 for a zero row),
    codes of (x / s) after clamping; also the codes a reciprocal multiply gives."""
    xf = x.float()
    s = xf.abs().amax(dim=1) / torch.tensor(DIVISOR, dtype=torch.float32)
    s = torch.where(s == 0, torch.ones_like(s), s)
    div = _codes(xf / s[:, None])
    mul = _codes(xf * (torch.ones_like(s) / s)[:, None])
    return div, s.numpy(), mul


def _tie_rows(exponents=(-20, 0, 30)) -> torch.Tensor:
    """One row per (bf16 significand of the row maximum a, binade): a itself,
    then every positive bf16 x in [a 2^-14, a) and its negative; zero padded."""
    pos = (np.arange(1, 0x7F80, dtype=np.uint32) << 16).view(np.float32)
    rows = []
    for e in exponents:
        for sig in range(128):
            a = np.float32(np.ldexp(1.0 + sig / 128.0, e))
            x = pos[(pos < a) & (pos >= a * np.float32(2.0 ** -14))]
            rows.append(np.concatenate([[a], x, -x]).astype(np.float32))
    k = -(-max(len(r) for r in rows) // 8) * 8
    out = np.zeros((len(rows), k), dtype=np.float32)
    for i, r in enumerate(rows):
        out[i, :len(r)] = r
    return torch.from_numpy(out).to(torch.bfloat16)   # every value is a bf16 already


def _many_scales() -> torch.Tensor:
    """Rows whose maxima span 2^-40..2^40 (and subnormal / overflowing scales),
    other values log-uniform over 40 binades below: the GPU parity input of the
    row quantizer, generated here on the CPU."""
    g = np.random.default_rng(77)
    rows, k = 2048, 1024
    amax = np.ldexp(1.0 + g.random(rows), g.integers(-40, 41, rows))
    amax[:4] = [1e-39, 3e-36, 2.0 ** 126, 3.0e38]
    mag = np.exp2(-40.0 * g.random((rows, k))) * amax[:, None]
    x = np.where(g.random((rows, k)) < 0.5, -mag, mag)
    x[np.arange(rows), g.integers(0, k, rows)] = amax
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)


def _check_rowwise(orc, x: torch.Tensor, min_sensitive: int):
    div, s, mul = _torch_rowwise(x)
    sensitive = int((div != mul).sum())
    assert sensitive >= min_sensitive, f"only {sensitive} reciprocal-sensitive elements"
    q, s_o = orc.quantize_rowwise(synthetic.bits(x))
    assert np.array_equal(s_o.view(np.uint32), s.view(np.uint32))
    bad = np.argwhere(q != div)
    assert bad.size == 0, f"{len(bad)} codes differ from fp32 division, first at {bad[0]}"


def test_rowwise_quotient_is_ieee_division_at_ties(orc):
    _check_rowwise(orc, _tie_rows(), min_sensitive=600)


def test_rowwise_quotient_is_ieee_division_many_scales(orc):
    _check_rowwise(orc, _many_scales(), min_sensitive=1000)


def _static_scales():
    """A dozen non-power-of-two scales: six of the form fp32(a / 448) for row
    maxima whose ties separate division from a reciprocal multiply, six spread
    over the fp32 range."""
    tie = [np.float32(np.float64(a) / DIVISOR) for a in (1.078125, 1.1875, 1.4375, 1.65625, 1.859375, 1.984375)]
    other = [np.float32(v) for v in (3.0e-30, 7.1e-9, 0.3, 1.7, 5.5e5, 2.9e33)]
    return tie + other


def test_static_quotient_is_ieee_division(orc):
    """Every finite bf16 value (both signs) at each scale: codes equal torch's
    fp32 division then E4M3; some elements change under x * (1/s)."""
    bits = np.arange(0, 0x7F80, dtype=np.uint32)
    pos = (bits << 16).view(np.float32)
    x = torch.from_numpy(np.concatenate([pos, -pos]).reshape(2, -1)).to(torch.bfloat16)
    sensitive = 0
    for s in _static_scales():
        st = torch.tensor(s, dtype=torch.float32)
        div = _codes(x.float() / st)
        sensitive += int((div != _codes(x.float() * (torch.tensor(1.0) / st))).sum())
        q = orc.quantize_static(synthetic.bits(x), s)
        bad = np.argwhere(q != div)
        assert bad.size == 0, f"scale {s}: {len(bad)} codes differ, first at {bad[0]}"
    assert sensitive >= 60, f"only {sensitive} reciprocal-sensitive elements"
