"""B200-native scaled FP8 / MXFP8 GEMM and quantizers (sm_100a).

The compute lives in ``libfp8mm.so`` (hand-written CUDA: tcgen05 / TMA / TMEM
GEMMs and vectorised quantizers) behind the C ABI of ``include/fp8mm.h``;
``fp8mm`` is its thin Python binding and ``synthetic`` draws the seeded
workload inputs.

Typical use (all tensors on the current CUDA device, the current stream)::

    import mxfp8_block_scaled_fp8_b200 as fp8mm
    # per-token / per-channel scales (DeepGEMM-style fp8_gemm)
    qa, sa = fp8mm.fp8_quantize_rowwise(a_bf16)          # [m, k] codes, [m] fp32
    qb, sb = fp8mm.fp8_quantize_rowwise(w_bf16)          # weight as [n, k]
    c = fp8mm.fp8_gemm(qa, qb, sa, sb)                   # bf16 [m, n]
    # MXFP8: 1x32 UE8M0 block scales in the library's scale layout
    qw, sfw = fp8mm.mxfp8_quantize(w_bf16)               # once, at load
    qx, sfx = fp8mm.mxfp8_quantize(x_bf16)               # per call
    c = fp8mm.mxfp8_gemm(qx, sfx, qw, sfw)
    # decode (m <= 64): bf16 activation in, K split over the SMs in a zeroed
    # workspace that later calls reuse (the counters are left at zero)
    ws = torch.zeros(fp8mm.quantize_gemm_workspace_bytes(m, n, k), dtype=torch.uint8, device="cuda")
    c = fp8mm.mxfp8_quantize_gemm(x_bf16, qw, sfw, workspace=ws, weights_ready=True)

``workspace_bytes`` also sizes the workspace that lets long-K GEMMs with
m > 64 split the K range of the tiles of their last, partly filled wave over
SM pairs (0 when a shape never splits; ``pair_split_plan`` tells how a shape
splits); ``sf_to_canonical`` / ``sf_from_canonical`` convert scales to and
from the row-major [rows, k / 32] tensor.  For activations of a few token
rows, ``mxfp8_quantize_8x4`` writes the scales in the small-M layout (rows
padded to 8 instead of 128) that ``mxfp8_gemm(..., sf_a_8x4=True)`` reads.
"""
from .fp8mm import (  # noqa: F401
    Fp8mmError, KERNEL_AUTO, concat_mla_k, KERNEL_SMALL_M, KERNEL_TILED, KERNEL_TILED_1SM, KERNEL_TILED_2SM, KERNEL_TILED_1SM_N128, fp8_gemm, fp8_gemm_e4m3_out, fp8_quantize_rowwise,
    fp8_quantize_static, fp8_tensor_scale, last_device_error,
    mxfp8_gemm, mxfp8_quantize, mxfp8_quantize_8x4, mxfp8_quantize_gemm, selftest_wait_timeout, sf_bytes,
    sf_from_canonical, sf_offset, sf_to_canonical, sf8x4_bytes, sf8x4_offset,
    pair_split_plan, quantize_gemm_workspace_bytes, version, workspace_bytes,
)
