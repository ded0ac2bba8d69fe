"""Helpers shared by the GPU parity tests (no method arithmetic here)."""
import numpy as np
import torch

# GEMM tolerance: relative Frobenius error <= 5e-3, and every element within
# 1e-2 * rms(oracle) of the float64 oracle *after* the BF16 output rounding the
# method prescribes: |got - ref| <= 1e-2 * rms(ref) + ulp_bf16(ref) / 2.  (The
# rounding of an exact result to BF16 alone can exceed 1e-2 * rms on elements
# above ~2.6 rms, so the bound without that term holds for no BF16 output.)
REL_FRO_TOL = 5e-3
ELEM_RMS_TOL = 1e-2


def half_ulp_bf16(ref: np.ndarray) -> np.ndarray:
    """Half a BF16 unit in the last place at |ref| (8 significant bits)."""
    _, e = np.frexp(np.abs(ref))  # |ref| = f * 2^e, f in [0.5, 1)
    return np.ldexp(1.0, e - 9) * (ref != 0)


def has_gpu() -> bool:
    return torch.cuda.is_available()


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> host uint16 bit patterns."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def u8(t: torch.Tensor) -> np.ndarray:
    """float8 / uint8 tensor -> host uint8 bytes."""
    return t.detach().contiguous().cpu().view(torch.uint8).numpy()


def scale_bytes(t: torch.Tensor) -> np.ndarray:
    """Scale array (float32 or uint8) -> host bytes, for bitwise comparison."""
    return t.detach().contiguous().cpu().view(torch.uint8).numpy()


def to_f64(d: torch.Tensor) -> np.ndarray:
    return d.detach().float().cpu().numpy().astype(np.float64)


def assert_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    diff = got - ref
    rel = np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300)
    rms = np.sqrt(np.mean(ref * ref))
    excess = np.abs(diff) - (ELEM_RMS_TOL * rms + half_ulp_bf16(ref))
    worst = excess.max() if diff.size else -1.0
    assert rel <= REL_FRO_TOL, f"{what}: relative Frobenius error {rel:.3e}"
    assert worst <= 0.0, f"{what}: element off by {worst:.3e} beyond 1e-2*rms + ulp/2 (rms {rms:.3e})"
    return rel, float(np.abs(diff).max() / max(rms, 1e-300))


def sample_indices(n: int, k: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    idx = rng.choice(n, size=min(k, n), replace=False)
    idx[0] = n - 1  # always include the last row/column (ragged tail)
    return np.sort(idx)
