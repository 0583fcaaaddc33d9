"""Shared helpers for the GPU parity tests: tensor transfer and the tolerances.

Tolerances (the GPU path computes in fp32; the oracle is fp64):
* fp32 activations: max_i |g_i - o_i| / max(|o_i|, rms(o)) <= 1e-4 (relative error,
  floored at the output RMS where the output crosses zero).
* bf16 activations (fp32 state, bf16 output): |g_i - o_i| <= 2e-2 * rms(o) + 2^-8 |o_i|.
  The 2e-2 * rms bound covers the arithmetic; the second term is the output's own
  round-to-nearest into bf16 (at most 2^-8 of the value). It is needed because |y|
  reaches 25-50 x rms(y) with these inputs, where rounding the exact result to bf16
  alone moves it by up to ~0.08 x rms. In addition every bf16 output must lie within
  one bf16 ulp of the oracle value rounded to bf16 (``assert_bf16_ulp``).
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


BF16_ROUND = 2.0 ** -8   # max relative error of round-to-nearest into bf16


def err_metric(g, o, dtype):
    """fp32: max relative error (floored at rms). bf16: max over elements of
    (|g - o| - 2^-8 |o|)_+ / rms(o), i.e. the error beyond the output's own rounding."""
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    if not o.size:
        return 0.0
    rms = float(np.sqrt(np.mean(o * o)))
    if dtype == "f32":
        den = np.maximum(np.abs(o), rms)
        den = np.where(den == 0, 1.0, den)
        return float(np.max(np.abs(g - o) / den))
    excess = np.maximum(np.abs(g - o) - BF16_ROUND * np.abs(o), 0.0)
    return float(np.max(excess) / (rms if rms > 0 else 1.0))


def plain_err(g, o):
    """max_i |g_i - o_i| / rms(o): the error as it is, rounding of the output included."""
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    if not o.size:
        return 0.0
    rms = float(np.sqrt(np.mean(o * o)))
    return float(np.max(np.abs(g - o)) / (rms if rms > 0 else 1.0))


def max_bf16_ulp(g, o):
    """Largest distance of a bf16 output from the rounded oracle value, in bf16 ulps."""
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    if not o.size:
        return 0.0
    ob = _bf16_round(o.astype(np.float32))
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ob), 2.0 ** -126))) - 7)
    return float(np.max(np.abs(g - ob) / ulp))


def _bf16_round(x):
    from mamba_selective_scan_sm_b200.synth import round_bf16
    return round_bf16(np.asarray(x, dtype=np.float32)).astype(np.float64)


def assert_bf16_ulp(g, o, what=""):
    """Every bf16 output within one bf16 ulp of bf16(o), or within 1e-4 * rms(o) where
    cancellation leaves |o| far below the output's scale."""
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    ob = _bf16_round(o.astype(np.float32))
    mag = np.maximum(np.abs(ob), 2.0 ** -126)
    ulp = 2.0 ** (np.floor(np.log2(mag)) - 7)
    floor = 1e-4 * float(np.sqrt(np.mean(o * o))) if o.size else 0.0
    bad = np.abs(g - ob) > np.maximum(ulp * (1 + 1e-9), floor)
    assert not np.any(bad), (f"{what}: {int(bad.sum())} outputs more than 1 bf16 ulp from the "
                             f"rounded oracle, worst {np.max(np.abs(g - ob) / ulp):.2f} ulp")


def assert_close(g, o, dtype, what=""):
    """The tolerance check; reports (pytest -s) the plain max |g - o| / rms(o) beside the
    metric the tolerance bounds (for bf16: the error beyond the output's own rounding)."""
    e = err_metric(g, o, dtype)
    tol = F32_TOL if dtype == "f32" else BF16_TOL
    plain = plain_err(g, o)
    print(f"{what}: max|g-o|/rms {plain:.3e}, "
          + (f"max rel {e:.3e}" if dtype == "f32" else
             f"beyond bf16 rounding {e:.3e}, worst {max_bf16_ulp(g, o):.2f} bf16 ulp"))
    assert np.all(np.isfinite(np.asarray(g, dtype=np.float64))), f"{what}: non-finite output"
    assert e <= tol, f"{what}: error {e:.3e} > {tol:.0e} (max|g-o|/rms {plain:.3e})"
    return e


def assert_close_out(g, o, dtype, what="", ulp=True):
    """Output check: the tolerance, plus (bf16) the one-ulp agreement."""
    e = assert_close(g, o, dtype, what)
    if dtype == "bf16" and ulp:
        assert_bf16_ulp(g, o, what)
    return e


def state_close(g, o, what=""):
    """Final states are fp32 on both dtypes: fp32 rule."""
    return assert_close(g, o, "f32", what)
