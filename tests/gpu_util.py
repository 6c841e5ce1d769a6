"""Shared helpers for the GPU parity tests (the oracle side always quantizes
and multiplies on its own; nothing it consumes comes from the GPU)."""
import numpy as np
import torch

# Acceptance bar of the scaled GEMM, on the dequantized-operand product:
#   |c - c_ref| <= 4e-3 * sum_k |a_k b_k| + 2^-8 |c_ref|  per element, and
#   ||c - c_ref||_F / ||c_ref||_F <= 2e-3.
ABS_BOUND_FACTOR = 4e-3
REL_FACTOR = 2.0 ** -8
FRO_LIMIT = 2e-3


def require_gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    major, _ = torch.cuda.get_device_capability()
    assert major == 10, "GPU tests need an sm_100 (B200) device"


def to_dev(t: torch.Tensor) -> torch.Tensor:
    return t.to("cuda", non_blocking=False)


def check_gemm(c_gpu: torch.Tensor, c_ref: np.ndarray, bound: np.ndarray, label: str = ""):
    c = c_gpu.float().cpu().numpy().astype(np.float64)
    assert c.shape == c_ref.shape, (c.shape, c_ref.shape)
    assert np.all(np.isfinite(c)), f"{label}: non-finite output"
    err = np.abs(c - c_ref)
    lim = ABS_BOUND_FACTOR * bound + REL_FACTOR * np.abs(c_ref)
    ratio = np.where(lim > 0, err / np.where(lim > 0, lim, 1.0), np.where(err > 0, np.inf, 0.0))
    worst = float(ratio.max()) if ratio.size else 0.0
    denom = np.linalg.norm(c_ref)
    fro = float(np.linalg.norm(c - c_ref) / denom) if denom > 0 else float(np.linalg.norm(c))
    i = np.unravel_index(int(np.argmax(ratio)), ratio.shape) if ratio.size else None
    info = (f"{label}: worst tol ratio {worst:.3g} at {i} (c={c[i] if i else None}, ref={c_ref[i] if i else None}), "
            f"rel-Fro {fro:.3g}, max abs {float(err.max()) if err.size else 0:.3g}, mean abs "
            f"{float(err.mean()) if err.size else 0:.3g}")
    assert worst <= 1.0, info
    assert fro <= FRO_LIMIT, info
    return worst, fro


def sf_canonical_from_layout(sf: np.ndarray, rows: int, k: int) -> np.ndarray:
    """Read the library's scale layout into canonical [rows, k/32], from the
    layout formula written out here (not the library's own helper)."""
    n_kc = -(-k // 128)
    nkb = k // 32
    r = np.arange(rows)[:, None]
    b = np.arange(nkb)[None, :]
    off = ((r // 128) * n_kc + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (b % 4)
    return sf[off]


def sf_layout_from_canonical(canon: np.ndarray, rows: int, k: int) -> np.ndarray:
    n_kc = -(-k // 128)
    rows_pad = -(-rows // 128) * 128
    out = np.zeros(rows_pad * n_kc * 4, dtype=np.uint8)
    nkb = k // 32
    r = np.arange(rows)[:, None]
    b = np.arange(nkb)[None, :]
    off = ((r // 128) * n_kc + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (b % 4)
    out[off] = canon
    return out
