"""Shared helpers for the GPU parity tests: tensor transfer and the tolerances.

Tolerances (the arithmetic is fp32 on both the GPU path and, up to rounding, the
fp64 oracle's definition):
* fp32 activations: max_i |g_i - o_i| / max(|o_i|, rms(o)) <= 1e-4 (relative error,
  floored at the output RMS where the output crosses zero).
* bf16 activations (fp32 state): max_i |g_i - o_i| <= 2e-2 * rms(o).
"""
import numpy as np
import torch

F32_TOL = 1e-4
BF16_TOL = 2e-2


def dev(x, dtype="f32"):
    """numpy (fp32 values; bf16-representable when dtype='bf16') -> CUDA tensor."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    if dtype == "bf16":
        t = t.to(torch.bfloat16)          # exact: the values are bf16-representable
    return t


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def err_metric(g, o, dtype):
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    rms = float(np.sqrt(np.mean(o * o))) if o.size else 0.0
    if dtype == "f32":
        den = np.maximum(np.abs(o), rms)
        den = np.where(den == 0, 1.0, den)
        return float(np.max(np.abs(g - o) / den)) if o.size else 0.0
    return float(np.max(np.abs(g - o)) / (rms if rms > 0 else 1.0)) if o.size else 0.0


def assert_close(g, o, dtype, what=""):
    e = err_metric(g, o, dtype)
    tol = F32_TOL if dtype == "f32" else BF16_TOL
    assert np.all(np.isfinite(np.asarray(g, dtype=np.float64))), f"{what}: non-finite output"
    assert e <= tol, f"{what}: error {e:.3e} > {tol:.0e}"
    return e


def state_close(g, o, what=""):
    """Final states are fp32 on both dtypes: fp32 rule."""
    return assert_close(g, o, "f32", what)
