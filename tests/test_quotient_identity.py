"""The per-row E4M3 quantizer divides each element by the row scale with
Markstein's residual correction instead of a division per element; the E4M3
code of the quotient must still be that of the IEEE fp32 quotient x / s (page
"从 DeepGEMM 到 vLLM", listing 3, per-row scale rule).  This host-side test
checks that identity exhaustively over significands with plain IEEE fp32
arithmetic (tests/quotient_identity.c); the GPU tests compare the kernel's
codes with the oracle."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_markstein_quotient_is_the_ieee_quotient(tmp_path):
    exe = tmp_path / "quotient_identity"
    subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                    os.path.join(HERE, "quotient_identity.c"), "-o", str(exe), "-lm", "-lpthread"], check=True)
    threads = max(1, min(32, os.cpu_count() or 1))
    r = subprocess.run([str(exe), str(threads)], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "exhaustive: 4294967296 pairs, 0 mismatches" in r.stdout, r.stdout
