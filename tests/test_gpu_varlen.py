"""GPU parity of packed sequences (seq_starts): several sequences share the sequence
axis of one batch row. The definition, and so the oracle side, is each sequence
scanned alone (zero state, zero conv history) and the results concatenated; final
states and conv states per sequence."""
import numpy as np
import pytest
import torch

import oracle
import mamba_selective_scan_sm_b200 as ssm
from mamba_selective_scan_sm_b200 import synth
from tests.gpu_helpers import assert_bf16_ulp, assert_close, assert_close_out, dev, host, state_close

pytestmark = pytest.mark.gpu


def _starts(lengths):
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)


def _oracle(inp, starts, conv):
    ys, hs, cs = [], [], []
    for a, b in zip(starts[:-1], starts[1:]):
        sl = lambda k: np.ascontiguousarray(inp[k][..., a:b])
        if b > a:
            y, h = oracle.selective_scan(sl("u"), sl("delta"), inp["A"], sl("B"), sl("C"),
                                         inp["D"], sl("z"), inp["delta_bias"], True, False,
                                         inp["conv_w"] if conv else None,
                                         inp["conv_b"] if conv else None,
                                         return_final_state=True)
        else:
            y, h = np.zeros((1, inp["u"].shape[1], 0)), np.zeros((1,) + inp["A"].shape)
        ys.append(y)
        hs.append(h[0])
        if conv:
            cs.append(oracle.conv_tail(sl("u"), inp["conv_w"].shape[1])[0])
    return np.concatenate(ys, axis=-1), np.stack(hs), (np.stack(cs) if conv else None)


def _gpu(inp, dtype, starts, conv, chunks=0, packed=True):
    t = lambda k: dev(inp[k], dtype)
    f = lambda k: dev(inp[k])
    res = ssm.ssm_selective_scan_fwd(
        t("u"), t("delta"), f("A"), t("B"), t("C"), f("D"), t("z"), f("delta_bias"), True, False,
        f("conv_w") if conv else None, f("conv_b") if conv else None, return_final_state=True,
        num_chunks=chunks, return_conv_state=conv,
        seq_starts=torch.from_numpy(starts).cuda() if packed else None)
    torch.cuda.synchronize()
    return res


LENGTHS = {
    "mixed": [1, 2, 3, 31, 32, 33, 64, 100, 5],          # shorter than the conv, tile edges
    "tile-aligned": [32, 32, 64, 96],
    "one-long": [700],
    "with-empty": [40, 0, 7, 0, 0, 60],
    # sequences spanning several chunks (chunks with no start in them scan nothing) and
    # starts off the tile grid
    "spanning": [3, 500, 17, 1, 130],
}


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("conv", [True, False])
@pytest.mark.parametrize("chunks", [0, 3, 7])
@pytest.mark.parametrize("lengths", list(LENGTHS), ids=str)
@pytest.mark.parametrize("dstate", [16, 5])
def test_packed_sequences_match_oracle(dtype, conv, chunks, lengths, dstate):
    lens = LENGTHS[lengths]
    starts = _starts(lens)
    L = int(starts[-1])
    inp = synth.scan_inputs(1, 40, L, dstate, dtype, conv_width=4 if conv else 0, seed=60)
    res = _gpu(inp, dtype, starts, conv, chunks)
    yo, ho, co = _oracle(inp, starts, conv)
    assert_close_out(host(res[0]), yo, dtype, "y")
    state_close(host(res[1]), ho, "final states")
    if conv:
        np.testing.assert_array_equal(host(res[2]), co)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_one_packed_sequence_equals_the_plain_call(dtype):
    """A single packed sequence is the ordinary scan, bit for bit (both in one pass: the
    plain call would otherwise split this small grid into chunks with a carry, which
    changes the rounding order)."""
    inp = synth.scan_inputs(1, 40, 333, 16, dtype, conv_width=4, seed=61)
    a = _gpu(inp, dtype, _starts([333]), True, chunks=1)
    b = _gpu(inp, dtype, None, True, chunks=1, packed=False)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_packed_plain_path_matches_tma(monkeypatch):
    starts = _starts(LENGTHS["mixed"])
    inp = synth.scan_inputs(1, 40, int(starts[-1]), 16, "bf16", conv_width=4, seed=62)
    a = _gpu(inp, "bf16", starts, True)
    monkeypatch.setenv("SSM_NO_TMA", "1")
    b = _gpu(inp, "bf16", starts, True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_packed_wide_rows_four_lanes_per_channel():
    """Enough channels for the 4-lanes-per-channel split (d_inner >= 9472 at batch 1)."""
    starts = _starts([17, 45, 3, 99])
    inp = synth.scan_inputs(1, 9472, int(starts[-1]), 16, "bf16", conv_width=4, seed=63)
    res = _gpu(inp, "bf16", starts, True)
    chans = [0, 1, 31, 32, 4000, 9471]
    sub = dict(inp)
    for k in ("u", "delta", "z"):
        sub[k] = inp[k][:, chans]
    for k in ("A", "D", "delta_bias", "conv_w", "conv_b"):
        sub[k] = inp[k][chans]
    yo, ho, co = _oracle(sub, starts, True)
    assert_close_out(host(res[0])[:, chans], yo, "bf16", "y")
    state_close(host(res[1])[:, chans], ho, "final states")
    np.testing.assert_array_equal(host(res[2])[:, chans], co)
