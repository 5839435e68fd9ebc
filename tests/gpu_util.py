"""Helpers for the GPU parity tests: tolerance check against the fp64 oracle."""
import numpy as np
import torch

# Tolerances for bf16 inputs, fp32 accumulation and bf16 output.
MAX_ABS = 1e-2
REL_RMS = 2e-3
# Outputs of magnitude >= 4 sit where bf16 spacing is 2^-5 or wider: the correctly
# rounded value itself can miss MAX_ABS there (4.5095 rounds to 4.5, 0.0095 away;
# 4.326 to 4.3125, 0.0139 away).  Cases whose attention concentrates on a few keys
# use this per-element bound instead:
#   |gpu - ref| <= max(MAX_ABS, half_ulp_bf16(ref) + SLACK_REL * |ref| + SLACK_ABS),
# half_ulp_bf16(ref) being half the bf16 spacing of |ref|'s own binade (2^(e-8) for
# 2^e <= |ref| < 2^(e+1)) and the slack the fp32 accumulation's share.  Below
# |ref| = 4 the half ulp plus slack stays under MAX_ABS, so the bound is MAX_ABS.
SLACK_REL = 2.0 ** -12
SLACK_ABS = 1e-4


def half_ulp_bf16(x: np.ndarray) -> np.ndarray:
    """Half the bf16 spacing in the binade of |x| (x = 0: that of the smallest normal)."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(ax)) - 8.0)


def bf16_scaled_bound(ref: np.ndarray) -> np.ndarray:
    return np.maximum(MAX_ABS, half_ulp_bf16(ref) + SLACK_REL * np.abs(ref) + SLACK_ABS)


def as_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def parity(gpu: torch.Tensor, ref: np.ndarray, what: str = "", bf16_scaled: bool = False):
    """Element-by-element comparison of a bf16 GPU result with the fp64 oracle."""
    g = as_f64(gpu).reshape(ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU output"
    err = np.abs(g - ref)
    if bf16_scaled:
        bound = bf16_scaled_bound(ref)
        worst = float((err / bound).max()) if err.size else 0.0
        assert worst <= 1.0, f"{what}: error {worst:.3f} x the bf16-scaled bound"
        err = np.where(err <= MAX_ABS, err, 0.0)  # checked above
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(g - ref)) / denom if denom > 0 else float(np.linalg.norm(g - ref))
    assert max_abs <= MAX_ABS, f"{what}: max-abs {max_abs:.3e} > {MAX_ABS}"
    assert rel <= REL_RMS, f"{what}: rel-RMS {rel:.3e} > {REL_RMS}"
    return max_abs, rel
