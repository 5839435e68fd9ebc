"""Helpers for the GPU parity tests: tolerance check against the fp64 oracle."""
import numpy as np
import torch

# Tolerances for bf16 inputs, fp32 accumulation and bf16 output.
MAX_ABS = 1e-2
REL_RMS = 2e-3
# Outputs of magnitude >= 4 sit where bf16 spacing is 2^-5: the correctly rounded
# value itself can miss MAX_ABS by up to half of that.  Stress cases whose
# attention concentrates on a few keys use this per-element bound instead:
# |gpu - ref| <= max(MAX_ABS, BF16_REL * |ref| + 1e-3), BF16_REL = half a bf16 ulp
# relative to the value, at most.
BF16_REL = 2.0 ** -8


def as_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def parity(gpu: torch.Tensor, ref: np.ndarray, what: str = "", bf16_scaled: bool = False):
    """Element-by-element comparison of a bf16 GPU result with the fp64 oracle."""
    g = as_f64(gpu).reshape(ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU output"
    err = np.abs(g - ref)
    if bf16_scaled:
        bound = np.maximum(MAX_ABS, BF16_REL * np.abs(ref) + 1e-3)
        worst = float((err / bound).max()) if err.size else 0.0
        assert worst <= 1.0, f"{what}: error {worst:.3f} x the bf16-scaled bound"
        err = np.where(err <= MAX_ABS, err, 0.0)  # checked above
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(g - ref)) / denom if denom > 0 else float(np.linalg.norm(g - ref))
    assert max_abs <= MAX_ABS, f"{what}: max-abs {max_abs:.3e} > {MAX_ABS}"
    assert rel <= REL_RMS, f"{what}: rel-RMS {rel:.3e} > {REL_RMS}"
    return max_abs, rel
