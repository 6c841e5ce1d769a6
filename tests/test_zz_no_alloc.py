"""The no-allocation small-M GEMM (for callers that cannot allocate device
memory: its split-K scratch lives in a fixed array inside the library) is
called through the C ABI, twice in a row, and each result is checked against
the CPU oracle with the same acceptance bar as the other GEMM tests; the
regular mxfp8_gemm entry point (caller-owned workspace) must meet the same bar
on the same inputs.  Collected last on purpose, and independent of every other
test."""
import ctypes

import pytest
import torch

import mxfp8_block_scaled_fp8_b200 as fp8mm
from mxfp8_block_scaled_fp8_b200 import fp8mm as binding
from mxfp8_block_scaled_fp8_b200 import synthetic
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _entry():
    lib = ctypes.CDLL(binding.LIB_PATH)
    fn = lib.mxfp8_gemm_small_m_noalloc
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    fn.argtypes = [P, P, P, P, I64, I64, I64, P, I64, P]
    fn.restype = ctypes.c_int
    return fn


def _oracle(x_cpu, w_cpu):
    """c_ref and sum_k |a_k b_k| of the dequantized operands, from the CPU oracle
    (which quantizes the same bf16 inputs itself)."""
    import oracle
    qx, sfx = oracle.mx_quantize(synthetic.bits(x_cpu))
    qw, sfw = oracle.mx_quantize(synthetic.bits(w_cpu))
    return oracle.gemm_mx(qx, sfx, qw, sfw)


CASES = [  # (m, n, k, label)
    (1, 6144, 4096, "qkv m=1"),
    (8, 14336, 4096, "up m=8"),
    (64, 4096, 14336, "down m=64"),
    (17, 130, 4128, "ragged"),
    # 256 weight tiles, but the scratch holds 127 CTAs of 64 tokens: most CTAs
    # cover parts of three tiles (a partial, whole tiles, a partial)
    (64, 32768, 4096, "more tiles than CTAs"),
]


@pytest.mark.parametrize("m,n,k,label", CASES, ids=[c[3] for c in CASES])
def test_no_alloc_matches_regular_entry_point(m, n, k, label):
    gu.require_gpu()
    fn = _entry()
    x_cpu = synthetic.random_bf16((m, k), seed=100 + m)
    w_cpu = synthetic.random_bf16((n, k), seed=200 + n, sigma=0.02)
    qx, sfx = fp8mm.mxfp8_quantize(x_cpu.cuda())
    qw, sfw = fp8mm.mxfp8_quantize(w_cpu.cuda())
    ws = torch.zeros(fp8mm.workspace_bytes(m, n, k), dtype=torch.uint8, device="cuda")
    c_regular = fp8mm.mxfp8_gemm(qx, sfx, qw, sfw, workspace=ws)
    torch.cuda.synchronize()
    c_ref, bound = _oracle(x_cpu, w_cpu)
    gu.check_gemm(c_regular, c_ref, bound, f"regular entry point, {label}")
    stream = torch.cuda.current_stream().cuda_stream
    outs = []
    for _ in range(2):                                     # two calls in a row share the scratch
        c = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = fn(qx.data_ptr(), sfx.data_ptr(), qw.data_ptr(), sfw.data_ptr(), m, n, k, c.data_ptr(), n, stream)
        assert st == 0, f"status {st}"
        torch.cuda.synchronize()
        gu.check_gemm(c, c_ref, bound, f"no-alloc vs oracle, {label}")
        outs.append(c)
    assert torch.equal(outs[0], outs[1])
    assert fp8mm.last_device_error() == 0


def test_no_alloc_rejects_what_does_not_fit():
    gu.require_gpu()
    fn = _entry()
    dummy = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    p = dummy.data_ptr()
    assert fn(p, p, p, p, 65, 128, 128, p, 128, None) == 2              # m > 64
    assert fn(p, p, p, p, 8, 128 * 16385, 128, p, 128 * 16385, None) == 6   # more tiles than counters
