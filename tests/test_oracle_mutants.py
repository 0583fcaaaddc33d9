"""The oracle pins must catch plausible slips.

Each case plants one mistake in a temporary copy of the oracle's C source (on
the CPU, never in the CUDA path), builds it, points the oracle module at the
mutant library and runs every pin in ``test_oracle_pins``; at least one pin must
fail. The committed oracle itself is untouched.
"""
import itertools
import os

import numpy as np
import subprocess
import tempfile

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

# (name, text in oracle.c, replacement, occurrence: None = all)
MUTANTS = [
    ("skip term dropped", "if (Dv) y += Dv[d] * ut;", "", None),
    ("skip term outside the gate",
     "if (Dv) y += Dv[d] * ut;\n                if (zr) y *= silu(zr[t]);",
     "if (zr) y *= silu(zr[t]);\n                if (Dv) y += Dv[d] * ut;", None),
    ("decay sign flipped", "exp(dl * A[d * N + n])", "exp(-dl * A[d * N + n])", None),
    ("delta missing from the decay", "exp(dl * A[d * N + n])", "exp(A[d * N + n])", None),
    ("delta missing from dBu", "double dBu = dl * Br[n * bn + t * bt] * ut;",
     "double dBu = Br[n * bn + t * bt] * ut;", None),
    ("B and C swapped", "dl * Br[n * bn + t * bt] * ut", "dl * Cr[n * bn + t * bt] * ut", None),
    ("B read transposed", "dl * Br[n * bn + t * bt] * ut", "dl * Br[t * N + n] * ut", None),
    ("readout before the update",
     "h[n] = dA * h[n] + dBu;\n                    y += Cr[n * bn + t * bt] * h[n];",
     "y += Cr[n * bn + t * bt] * h[n];\n                    h[n] = dA * h[n] + dBu;", None),
    ("time-invariant B read as (N, D)", "bc_shared ? Bm + d * N : Bm + b * N * L",
     "bc_shared ? Bm + d : Bm + b * N * L", None),
    ("time-invariant B and C read as (N, D) matrices",
     "const double* Br = bc_shared ? Bm + d * N : Bm + b * N * L;\n"
     "            const double* Cr = bc_shared ? Cm + d * N : Cm + b * N * L;\n"
     "            const long bn = bc_shared ? 1 : L,",
     "const double* Br = bc_shared ? Bm + d : Bm + b * N * L;\n"
     "            const double* Cr = bc_shared ? Cm + d : Cm + b * N * L;\n"
     "            const long bn = bc_shared ? D : L,", None),
    ("conv taps reversed", "long s = t - (W - 1) + k;", "long s = t - k;", None),
    ("fused conv taps reversed", ": t - (conv_width - 1) + k;", ": t - k;", None),
    ("reverse conv uses forward taps", "t + (conv_width - 1) - k :", "t - (conv_width - 1) + k :",
     None),
    ("conv bias dropped", "double acc = conv_b ? conv_b[d] : 0.0;", "double acc = 0.0;", None),
    ("softplus replaced by exp", "return log1p(exp(x));", "return exp(x);", None),
    ("bias added after softplus",
     "double dl = dr[t] + (delta_bias ? delta_bias[d] : 0.0);\n"
     "                if (delta_softplus) dl = softplus(dl);",
     "double dl = dr[t];\n                if (delta_softplus) dl = softplus(dl);\n"
     "                dl += (delta_bias ? delta_bias[d] : 0.0);", None),
    ("silu replaced by sigmoid", "return v / (1.0 + exp(-v));", "return 1.0 / (1.0 + exp(-v));",
     None),
    ("decode conv window shifted the wrong way",
     "for (int k = 0; k < conv_width - 1; ++k) cs[k] = cs[k + 1];\n"
     "                cs[conv_width - 1] = xt;",
     "for (int k = conv_width - 1; k > 0; --k) cs[k] = cs[k - 1];\n"
     "                cs[0] = xt;", None),
    ("decode dt bias dropped", "double dl = dt[bd] + (dt_bias ? dt_bias[d] : 0.0);",
     "double dl = dt[bd];", None),
    ("decode skip term dropped", "if (Dv) y += Dv[d] * xc;", "", None),
    ("conv history read in reverse order", "(conv_width - 1) + s]", "-1 - s]", None),
    ("conv history ignored", "else if (s < 0 && !reverse && conv_hist)", "else if (0 && conv_hist)",
     None),
    ("initial state ignored", "h[n] = h0 ? h0[(b * D + d) * N + n] : 0.0;", "h[n] = 0.0;", None),
]


def _expand(fn):
    marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
    if not marks:
        return [{}]
    axes = []
    for m in marks:
        names = [n.strip() for n in m.args[0].split(",")]
        vals = [v if len(names) > 1 else (v,) for v in m.args[1]]
        axes.append([dict(zip(names, v)) for v in vals])
    out = []
    for combo in itertools.product(*axes):
        d = {}
        for c in combo:
            d.update(c)
        out.append(d)
    return out


PINS = [(name, fn, kw) for name, fn in vars(pins).items()
        if name.startswith("test_") and callable(fn) for kw in _expand(fn)]


def _failing_pins(lib):
    saved = oracle._lib
    oracle._lib = lib
    failed = []
    try:
        for name, fn, kw in PINS:
            try:
                fn(**kw)
            except AssertionError:
                failed.append(name)
            except Exception:            # a crash in a mutant also counts as caught
                failed.append(name + " (error)")
    finally:
        oracle._lib = saved
    return failed


def test_unmutated_oracle_passes_every_pin():
    assert _failing_pins(oracle._load()) == []


@pytest.mark.parametrize("name,old,new,occ", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, occ, tmp_path):
    src = open(SRC).read()
    assert old in src, f"mutation anchor not found: {name}"
    mutated = src.replace(old, new)
    c = tmp_path / "mut.c"
    so = tmp_path / "libmut.so"
    c.write_text(mutated)
    subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-std=c99",
                           "-shared", "-fPIC", "-o", str(so), str(c), "-lm"])
    failed = _failing_pins(oracle.load_library(str(so)))
    assert failed, f"no pin caught the planted mistake: {name}"


def test_head_mapping_slip_is_caught(monkeypatch):
    """A plausible slip in the per-head expansion (heads interleaved across channels
    instead of contiguous) fails the dual-form pin."""
    def wrong(A, dim, N):
        A = np.asarray(A, dtype=np.float64)
        if A.ndim == 2:
            return A
        return np.tile(A, dim // A.shape[0])[:, None] * np.ones((1, N))
    monkeypatch.setattr(oracle, "head_A", wrong)
    with pytest.raises(AssertionError):
        pins.test_scalar_A_per_head_equals_ssd_dual_form(4, False)


def _swapped_bidir(swap):
    """selective_scan_bidir with the named parameters exchanged between the directions."""
    real = oracle.selective_scan_bidir

    def wrong(u, delta, A, B, C, D, z, delta_bias, A_rev, D_rev, delta_bias_rev, *a, **kw):
        if "A" in swap:
            A, A_rev = A_rev, A
        if "D" in swap:
            D, D_rev = D_rev, D
        if "bias" in swap:
            delta_bias, delta_bias_rev = delta_bias_rev, delta_bias
        return real(u, delta, A, B, C, D, z, delta_bias, A_rev, D_rev, delta_bias_rev, *a, **kw)
    return wrong


@pytest.mark.parametrize("swap", [("A", "D", "bias"), ("A",), ("bias",), ("A", "D"), ("D", "bias")],
                         ids=["all", "A", "bias", "A_and_D", "D_and_bias"])
def test_bidirectional_direction_swap_is_caught(swap, monkeypatch):
    """Routing a direction's A or dt bias to the other direction fails a pin. (D
    alone has no wrong routing: the two skip terms add up to (D + D_rev) * u under the
    shared gate, so exchanging only D leaves the sum unchanged.)"""
    monkeypatch.setattr(oracle, "selective_scan_bidir", _swapped_bidir(swap))
    assert _failing_pins(oracle._load()), f"no pin caught the exchanged {swap}"
