"""B200-native scaled FP8 / MXFP8 GEMM and quantizers (sm_100a).

The compute lives in ``libfp8mm.so`` (hand-written CUDA: tcgen05 / TMA / TMEM
GEMMs and vectorised quantizers) behind the C ABI of ``include/fp8mm.h``;
``fp8mm`` is its thin Python binding and ``synthetic`` draws the seeded
workload inputs.
"""
from .fp8mm import (  # noqa: F401
    Fp8mmError, KERNEL_AUTO, concat_mla_k, KERNEL_SMALL_M, KERNEL_TILED, KERNEL_TILED_1SM, KERNEL_TILED_2SM, KERNEL_TILED_1SM_N128, fp8_gemm, fp8_gemm_e4m3_out, fp8_quantize_rowwise,
    fp8_quantize_static, fp8_tensor_scale, last_device_error,
    mxfp8_gemm, mxfp8_quantize, mxfp8_quantize_gemm, selftest_wait_timeout, sf_bytes, sf_from_canonical, sf_offset, sf_to_canonical,
    quantize_gemm_workspace_bytes, version, workspace_bytes,
)
