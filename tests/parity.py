"""Comparison helpers for the GPU parity tests (CUDA library vs fp64 oracle).

Tolerances for attention outputs, against the fp64 oracle evaluated on the
same bf16-rounded inputs: max-abs <= 2e-2 and relative L2 <= 5e-3.  The bf16
path rounds P to bf16 before PV and rounds the output to bf16 (relative
error ~2^-9 each), so the expected relative L2 is ~1-2e-3.  MSE results:
relative error <= 1e-5.
"""
import numpy as np
import torch

ATTN_MAX_ABS = 2e-2
ATTN_REL_L2 = 5e-3
MSE_REL = 1e-5


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def attn_errors(got: np.ndarray, want: np.ndarray):
    diff = got - want
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    denom = float(np.linalg.norm(want))
    rel = float(np.linalg.norm(diff)) / denom if denom > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_attn_close(got, want, what=""):
    got = to_f64(got) if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    max_abs, rel = attn_errors(got, want)
    assert max_abs <= ATTN_MAX_ABS and rel <= ATTN_REL_L2, \
        f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel


GUARD = 4096  # elements on each side


def guarded_empty(shape, dtype, device="cuda"):
    """An output tensor with NaN-patterned guard regions on both sides."""
    n = int(np.prod(shape))
    base = torch.full((n + 2 * GUARD,), float("nan"), dtype=dtype, device=device)
    return base, base[GUARD:GUARD + n].view(shape)


def check_guards(base: torch.Tensor):
    lo = base[:GUARD]
    hi = base[-GUARD:]
    assert torch.isnan(lo.float()).all() and torch.isnan(hi.float()).all(), "guard region overwritten"
