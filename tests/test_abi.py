"""The C-ABI library loads without a GPU, exports every function the header
declares, rejects bad arguments before touching CUDA, and its host-side scale
layout helpers agree with the layout formula the header documents."""
import ctypes
import os
import re
import shutil
import subprocess

import numpy as np
import pytest
import torch

import mxfp8_block_scaled_fp8_b200 as fp8mm
from mxfp8_block_scaled_fp8_b200 import fp8mm as binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8mm.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:[A-Za-z_][\w\s\*]*?)\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if not n.startswith("FP8MM")))


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(binding.LIB_PATH)
    declared = _declared()
    assert {"fp8_quantize_rowwise", "mxfp8_quantize", "fp8_gemm", "mxfp8_gemm"} <= set(declared)
    missing = [n for n in declared if not hasattr(lib, n)]
    assert not missing, missing
    assert set(binding._SIGNATURES) <= set(declared) | {"fp8mm_version"}


def test_version_and_status_strings():
    L = binding.lib()
    assert L.fp8mm_version() == 10000
    for s in range(0, 8):
        assert len(L.fp8mm_status_str(s)) > 0
    assert L.fp8mm_status_str(99) == b"unknown status"


def test_argument_errors_without_a_gpu():
    L = binding.lib()
    P = ctypes.c_void_p
    fake = 1 << 20                                             # never dereferenced
    # shapes
    assert L.fp8_gemm(P(fake), P(fake), 4, 4, 15, P(fake), P(fake), P(fake), 8, None, None) == 2
    assert L.mxfp8_gemm(P(fake), P(fake), P(fake), P(fake), 4, 4, 48, P(fake), 8, None, None) == 2
    assert L.fp8_quantize_rowwise(P(fake), 4, 12, 16, P(fake), 16, P(fake), None) == 2
    assert L.mxfp8_quantize(P(fake), 4, 40, 40, P(fake), 40, P(fake), None) == 2
    assert L.fp8_gemm(P(fake), P(fake), -1, 4, 16, P(fake), P(fake), P(fake), 8, None, None) == 2
    assert L.fp8_gemm(P(fake), P(fake), 4, 16, 16, P(fake), P(fake), P(fake), 8, None, None) == 2   # ldc < n
    # null pointers
    assert L.fp8_gemm(None, P(fake), 4, 4, 16, P(fake), P(fake), P(fake), 8, None, None) == 1
    assert L.mxfp8_gemm(P(fake), None, P(fake), P(fake), 4, 4, 32, P(fake), 8, None, None) == 1
    assert L.mxfp8_quantize(P(fake), 4, 32, 32, P(fake), 32, None, None) == 1
    # alignment
    assert L.fp8_gemm(P(fake + 8), P(fake), 4, 4, 16, P(fake), P(fake), P(fake), 8, None, None) == 3
    assert L.fp8_gemm(P(fake), P(fake), 4, 4, 16, P(fake), P(fake), P(fake + 1), 12, None, None) == 3
    assert L.mxfp8_quantize(P(fake), 4, 32, 36, P(fake), 32, P(fake), None) == 3
    # activation-quantizing decode GEMM
    Q = L.mxfp8_quantize_gemm
    assert Q(P(fake), 64, P(fake), P(fake), 65, 4, 64, P(fake), 8, None, None) == 2     # m > 64
    assert Q(P(fake), 64, P(fake), P(fake), 4, 4, 48, P(fake), 8, None, None) == 2     # k % 32
    assert Q(P(fake), 32, P(fake), P(fake), 4, 4, 64, P(fake), 8, None, None) == 2     # lda < k
    assert Q(P(fake), 68, P(fake), P(fake), 4, 4, 64, P(fake), 8, None, None) == 3     # lda % 8
    assert Q(P(fake + 8), 64, P(fake), P(fake), 4, 4, 64, P(fake), 8, None, None) == 3  # a alignment
    assert Q(P(fake), 64, P(fake), None, 4, 4, 64, P(fake), 8, None, None) == 1        # sf_b
    tiled = binding.Opts(None, 0, binding.KERNEL_TILED, 0, 0)
    assert Q(P(fake), 64, P(fake), P(fake), 4, 4, 64, P(fake), 8, ctypes.byref(tiled), None) == 2
    assert Q(None, 64, None, None, 0, 4, 64, None, 8, None, None) == 0                 # m == 0
    assert Q(P(fake), 64, P(fake), P(fake), 9, 4, 64, P(fake), 8, None, None) == 6      # m > 8 needs a workspace
    # per-tensor scale, static quantizer, E4M3-output GEMM, MLA key concatenation
    assert L.fp8_tensor_scale(P(fake), 4, 12, 16, P(fake), None) == 2                       # k % 8
    assert L.fp8_tensor_scale(P(fake), 4, 16, 16, None, None) == 1                          # scale
    assert L.fp8_quantize_static(P(fake), 4, 16, 16, None, P(fake), 16, None) == 1          # scale
    assert L.fp8_quantize_static(P(fake), 4, 16, 16, P(fake), P(fake + 4), 16, None) == 3   # q alignment
    assert L.fp8_quantize_static(None, 0, 16, 16, None, None, 16, None) == 0                # empty
    E = L.fp8_gemm_e4m3_out
    assert E(P(fake), P(fake), 4, 4, 15, P(fake), P(fake), P(fake), P(fake), 8, None, None) == 2      # k % 16
    assert E(P(fake), P(fake), 4, 4, 16, P(fake), P(fake), None, P(fake), 8, None, None) == 1         # scale_out
    assert E(P(fake), P(fake), 4, 4, 16, P(fake), P(fake), P(fake), P(fake + 1), 8, None, None) != 3  # any c alignment
    C = L.concat_mla_k
    assert C(P(fake), P(fake), P(fake), 2, 2, 128, 64, 3, 256, 128, 64, 0, 384, 192, None) == 2       # elem bytes
    assert C(P(fake), P(fake), P(fake), 2, 2, 120, 64, 1, 240, 120, 64, 0, 368, 184, None) == 3       # 120-byte rows
    assert C(P(fake + 8), P(fake), P(fake), 2, 2, 128, 64, 1, 256, 128, 64, 0, 384, 192, None) == 3   # base
    assert C(None, None, None, 0, 2, 128, 64, 1, 256, 128, 64, 0, 384, 192, None) == 0                # no tokens
    # kernel choices: 0..5 are known, others are rejected before any device work
    for bad in (-1, 6):
        o = binding.Opts(None, 0, bad, 0, 0)
        assert L.fp8_gemm(P(fake), P(fake), 4, 4, 16, P(fake), P(fake), P(fake), 8, ctypes.byref(o), None) == 2
        assert L.mxfp8_gemm(P(fake), P(fake), P(fake), P(fake), 4, 4, 32, P(fake), 8, ctypes.byref(o), None) == 2
        assert E(P(fake), P(fake), 4, 4, 16, P(fake), P(fake), P(fake), P(fake), 8, ctypes.byref(o), None) == 2
    assert binding.KERNEL_TILED_1SM_N128 == 5
    # empty problems are no-ops and need no device
    assert L.fp8_gemm(None, None, 0, 4, 16, None, None, None, 8, None, None) == 0
    assert L.mxfp8_quantize(None, 0, 64, 64, None, 64, None, None) == 0
    assert L.fp8_quantize_rowwise(None, 0, 64, 64, None, 64, None, None) == 0


def test_workspace_sizes():
    # 2 * G * 128 * NM floats (256-byte aligned) + one counter per 128-row tile
    assert fp8mm.workspace_bytes(64, 14336, 4096, 148) == 2 * 148 * 128 * 64 * 4 + 512
    assert fp8mm.workspace_bytes(1, 4096, 14336, 148) == 2 * 148 * 128 * 16 * 4 + 256
    # m > 64 and K >= 8192 (64 slabs of 128): the paired kernel's K split, on a host without a GPU for
    # 148 SMs (74 pairs), whatever the tile count: room for one split part per pair, 128 x 256 fp32 per CTA
    # rank, then 2 counters per pair (256-byte rounded); shorter K is never split
    part = 128 * 256 * 4
    for shape in [(65, 4096, 8192), (512, 2048, 8192), (2048, 512, 16384), (2048, 1024, 8192),
                  (8192, 22016, 8192), (8192, 2048, 8192)]:
        assert fp8mm.workspace_bytes(*shape) == 74 * 2 * part + 768, shape
    assert fp8mm.workspace_bytes(2048, 1024, 4096) == 0                              # 32 K slabs
    assert fp8mm.workspace_bytes(65, 4096, 4096) == 0
    assert fp8mm.workspace_bytes(8, 128, 128, 148) == 2 * 1 * 128 * 16 * 4 + 256   # clamped to 1 unit
    # the small-M kernel's automatic CTA count (a host without a GPU counts 148 SMs), read back from the
    # partials' size: tile-aligned counts (s CTAs per 128-row weight tile, s dividing its K slabs) where one
    # fits within 75 % (16-token tiles) or 60 % (larger) of the default, else one or two per SM
    def auto_ctas(m, n, k):
        nm = 16 if m <= 16 else 32 if m <= 32 else 48 if m <= 48 else 64
        tickets = -(-(-(-n // 128) * 4) // 256) * 256
        return (fp8mm.workspace_bytes(m, n, k) - tickets) // (2 * 128 * nm * 4)
    expected = {(1, 14336, 4096): 224, (8, 14336, 4096): 224, (32, 14336, 4096): 224, (64, 14336, 4096): 224,
                (1, 4096, 14336): 256, (8, 4096, 14336): 256, (32, 4096, 14336): 256, (64, 4096, 14336): 256,
                (1, 6144, 4096): 192, (8, 6144, 4096): 192, (32, 6144, 4096): 192, (64, 6144, 4096): 192,
                (8, 1024, 2048): 32, (3, 200, 96): 2}
    got = {shape: auto_ctas(*shape) for shape in expected}
    assert got == expected
    # activation-quantizing GEMM: the same for m <= 8, plus the quantized activation and scales above
    assert fp8mm.quantize_gemm_workspace_bytes(8, 14336, 4096, 148) == fp8mm.workspace_bytes(8, 14336, 4096, 148)
    assert (fp8mm.quantize_gemm_workspace_bytes(33, 4096, 14336, 148) ==
            fp8mm.workspace_bytes(33, 4096, 14336, 148) + 33 * 14336 + fp8mm.sf_bytes(33, 14336))
    assert fp8mm.quantize_gemm_workspace_bytes(65, 4096, 4096, 148) == 0


def _layout_offset(rows, k, r, b):
    n_kc = -(-k // 128)
    return ((r // 128) * n_kc + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (b % 4)


@pytest.mark.parametrize("rows,k", [(1, 32), (130, 96), (256, 4096), (300, 160)])
def test_scale_layout_helpers(rows, k):
    assert fp8mm.sf_bytes(rows, k) == (-(-rows // 128) * 128) * (-(-k // 128)) * 4
    nkb = k // 32
    rng = np.random.default_rng(rows + k)
    canon = rng.integers(0, 255, size=(rows, nkb), dtype=np.uint8)
    sf = fp8mm.sf_from_canonical(torch.from_numpy(canon), rows, k).numpy()
    expect = np.zeros(fp8mm.sf_bytes(rows, k), dtype=np.uint8)
    for r in range(rows):
        for b in range(nkb):
            assert fp8mm.sf_offset(rows, k, r, b) == _layout_offset(rows, k, r, b)
            expect[_layout_offset(rows, k, r, b)] = canon[r, b]
    assert np.array_equal(sf, expect)
    assert np.array_equal(fp8mm.sf_to_canonical(torch.from_numpy(sf), rows, k).numpy(), canon)
    # every byte of the buffer belongs to exactly one (row, block) of the padded grid
    rp, kb4 = -(-rows // 128) * 128, -(-k // 128) * 4
    offs = sorted(fp8mm.sf_offset(rows, k, r, b) for r in range(rp) for b in range(kb4))
    assert offs == list(range(fp8mm.sf_bytes(rows, k)))
    assert fp8mm.sf_offset(rows, k, rp, 0) == -1


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(binding.Fp8mmError):
        binding.lib()


def test_sf8x4_layout_matches_header_formula():
    """The small-M layout: 32-byte atoms of 8 rows x 4 K-blocks, atom (r8, g) at
    (g * ceil(rows/8) + r8) * 32, byte (r % 8) * 4 + b % 4 inside; a bijection
    onto [0, sf8x4_bytes) over the padded rows and blocks."""
    for rows, k in [(1, 32), (5, 4096), (8, 160), (17, 14336), (64, 4128)]:
        rows8 = -(-rows // 8) * 8
        nb = -(-k // 128) * 4
        assert fp8mm.sf8x4_bytes(rows, k) == rows8 * nb
        seen = set()
        for r in range(rows8):
            for b in range(nb):
                off = fp8mm.sf8x4_offset(rows, k, r, b)
                atom = (b // 4) * (rows8 // 8) + r // 8
                assert off == atom * 32 + (r % 8) * 4 + b % 4
                seen.add(off)
        assert seen == set(range(rows8 * nb))
        assert fp8mm.sf8x4_offset(rows, k, rows8, 0) == -1 and fp8mm.sf8x4_offset(rows, k, 0, nb) == -1
    assert fp8mm.sf8x4_bytes(0, 64) == 0


def test_sf8x4_argument_errors_without_gpu():
    L = binding.lib()
    assert L.mxfp8_quantize_8x4(None, 4, 48, 48, None, 48, None, None) == 2      # k % 32
    assert L.mxfp8_quantize_8x4(None, 4, 64, 64, None, 64, None, None) == 1      # null pointers
    assert L.mxfp8_quantize_8x4(None, 0, 64, 64, None, 64, None, None) == 0      # nothing to do


def test_pair_split_plan():
    """The paired kernel's split plan: (K parts per split tile, tiles run whole).  The tiles of the last,
    partly filled wave of pairs are split into as many parts as fit the pairs it leaves (all tiles where
    they fill less than one wave), each of >= 16 K slabs of 128, <= 8 parts; none for m <= 64, K < 8192
    or whole waves."""
    plan = fp8mm.pair_split_plan
    assert plan(8192, 22016, 8192, 74) == (4, 2738)      # 2752 tiles: 37 waves + 14; 74 // 14 = 5 > 64 // 16
    assert plan(8192, 2048, 8192, 74) == (2, 222)        # 256 tiles: 3 waves + 34
    assert plan(2560, 2048, 8192, 74) == (4, 74)         # 80 tiles: 1 wave + 6
    assert plan(8192, 3584, 8192, 74) == (4, 444)        # 448 tiles: 6 waves + 4
    assert plan(8192, 9472, 8192, 74) == (1, 1184)       # 16 whole waves
    assert plan(8192, 3840, 8192, 74) == (2, 444)        # 480 tiles: 6 waves + 36; 74 // 36 = 2
    assert plan(8192, 4096, 8192, 74) == (1, 512)        # 512 tiles: 6 waves + 68; no room for 2 parts
    assert plan(512, 2048, 8192, 74) == (4, 0)           # 16 tiles, all split
    assert plan(2048, 1024, 8192, 74) == (2, 0)
    assert plan(300, 600, 8960, 74) == (4, 0)            # 70 slabs
    assert plan(2048, 512, 32768, 74) == (4, 0)          # 16 tiles: 74 // 16 = 4 parts of 64 slabs
    assert plan(512, 256, 32768, 74) == (8, 0)           # 2 tiles: capped at 8 parts
    assert plan(2048, 1024, 4096, 74) == (1, 32)         # 32 K slabs: never split
    assert plan(64, 4096, 8192, 74) == (1, 16)           # m <= 64: the small-M kernel's business
    assert plan(8192, 22016, 8192, 72) == (4, 2736)      # 72 pairs: 38 waves + 16; 72 // 16 = 4
    assert plan(0, 128, 128, 74) == (1, 0)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_opts_struct_layout_matches_the_header(tmp_path):
    """The binding's ctypes fp8mm_opts has the header's size and field offsets (compiled with gcc from
    include/fp8mm.h), so the options a Python caller sets are the ones the library reads."""
    src = tmp_path / "layout.c"
    fields = [name for name, _ in binding.Opts._fields_]
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "fp8mm.h"\nint main(void) {\n'
                   '  printf("size %zu\\n", sizeof(fp8mm_opts));\n'
                   + "".join(f'  printf("{f} %zu\\n", offsetof(fp8mm_opts, {f}));\n' for f in fields)
                   + "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True, text=True,
                                                        check=True).stdout.splitlines())
    assert int(out["size"]) == ctypes.sizeof(binding.Opts)
    for f in fields:
        assert int(out[f]) == getattr(binding.Opts, f).offset, f
