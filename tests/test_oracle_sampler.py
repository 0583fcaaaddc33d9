"""The oracle's channel sampler against the whole-array oracle (CPU only).

``oracle.scan_channels`` computes the oracle for a sample of (b, d) rows of a
full-size input; the full-size GPU parity tests and the bench's CPU baseline use
it. Here its rows must equal the same rows of one whole-array oracle call, for
every way it slices the inputs: per-state A and A per head, B/C per batch row and
time-invariant B/C, conv, reverse, bidirectional, final states.
"""
import numpy as np
import pytest

import oracle
from mamba_selective_scan_sm_b200 import synth

CHANS = [(0, 0), (1, 5), (2, 11), (1, 6), (0, 7)]


def _inputs(conv, bidir, heads, shared):
    return synth.scan_inputs(3, 12, 37, 8, "f32", 4 if conv else 0, bidir, seed=5,
                             a_heads=3 if heads else 0, bc_shared=shared)


def _whole(inp, conv, reverse, bidir):
    kw = dict(conv_w=inp.get("conv_w") if conv else None, conv_b=inp.get("conv_b") if conv else None)
    if bidir:
        y, hf, hr = oracle.selective_scan_bidir(
            inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["z"],
            inp["delta_bias"], inp["A_rev"], inp["D_rev"], inp["delta_bias_rev"], True,
            return_final_state=True, **kw)
        return y, hf, hr
    y, hf = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                  inp["z"], inp["delta_bias"], True, reverse,
                                  return_final_state=True, **kw)
    return y, hf, None


@pytest.mark.parametrize("heads", [False, True], ids=["A_per_state", "A_per_head"])
@pytest.mark.parametrize("shared", [False, True], ids=["BC_per_batch", "BC_time_invariant"])
@pytest.mark.parametrize("mode", ["forward", "reverse", "conv", "bidir"])
def test_sampler_rows_equal_whole_array_rows(heads, shared, mode):
    conv, reverse, bidir = mode == "conv", mode == "reverse", mode == "bidir"
    inp = _inputs(conv, bidir, heads, shared)
    y, hf, hr = _whole(inp, conv, reverse, bidir)
    res = oracle.scan_channels(inp, CHANS, reverse=reverse, conv=conv, final_state=True,
                               bidirectional=bidir)
    ys, hs = res[0], res[1]
    for i, (b, d) in enumerate(CHANS):
        np.testing.assert_array_equal(ys[i], y[b, d])
        np.testing.assert_array_equal(hs[i], hf[b, d])
        if bidir:
            np.testing.assert_array_equal(res[2][i], hr[b, d])


def test_sampler_sees_a_wrong_batch_row():
    """The check above can tell rows apart: B/C of another batch row give other outputs."""
    inp = _inputs(False, False, False, False)
    y, _, _ = _whole(inp, False, False, False)
    wrong = dict(inp)
    wrong["B"] = inp["B"][[1, 2, 0]]
    ys = oracle.scan_channels(wrong, CHANS)
    assert not np.allclose(ys[0], y[0, 0])
