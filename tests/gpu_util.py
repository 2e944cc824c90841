"""Shared helpers of the GPU parity tests (comparison metrics and the
tolerances that the tests apply)."""
import numpy as np
import torch

# Attention outputs: bf16 inputs, fp32 accumulation, bf16 output.
ATTN_MAX_ABS = 2e-2
ATTN_REL_L2 = 5e-3
LSE_ABS = 2e-3


def to_np_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_l2(got: np.ndarray, ref: np.ndarray) -> float:
    num = np.linalg.norm((got - ref).ravel())
    den = np.linalg.norm(ref.ravel())
    return float(num / den) if den > 0 else float(num)


def chain_lse_tol(q_norm, k_norm_max, scale):
    """LSE tolerance for chains that round rotated q and k to bf16 before the
    attention kernel: each factor carries a relative error <= 2^-9, so every
    score moves by at most 2^-8 * scale * |q| |k| (Cauchy-Schwarz), and a
    log-sum-exp moves by at most the largest score change."""
    return 2.0 ** -8 * scale * q_norm * k_norm_max + LSE_ABS


def assert_attn_close(out, ref_out, lse=None, ref_lse=None, what="", lse_tol=None):
    got = to_np_f64(out) if isinstance(out, torch.Tensor) else out
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref_out)
    assert err.max() <= ATTN_MAX_ABS, f"{what}: max-abs {err.max():.3e}"
    r = rel_l2(got, ref_out)
    assert r <= ATTN_REL_L2, f"{what}: rel-L2 {r:.3e}"
    if lse is not None:
        gl = to_np_f64(lse) if isinstance(lse, torch.Tensor) else lse
        fin = np.isfinite(ref_lse)
        assert np.array_equal(np.isfinite(gl), fin), f"{what}: lse finiteness differs"
        if fin.any():
            tol = np.broadcast_to(LSE_ABS if lse_tol is None else lse_tol, ref_lse.shape)[fin]
            e = np.abs(gl[fin] - ref_lse[fin])
            assert np.all(e <= tol), f"{what}: lse error {e.max():.3e} above its bound"


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, 2.0 ** (e - 7), 2.0 ** -133)
