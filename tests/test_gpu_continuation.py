"""GPU parity of a scan that continues a sequence: initial_state, conv_history and
conv_state_out of ssm_selective_scan_fwd, against the CPU oracle, element by element.

A prompt taken in pieces (each piece starting from the previous piece's final state
and conv state) must reproduce the one-piece scan, and decode steps must pick up
where a scan stopped."""
import numpy as np
import pytest
import torch

import oracle
import mamba_selective_scan_sm_b200 as ssm
from mamba_selective_scan_sm_b200 import synth
from tests.gpu_helpers import assert_bf16_ulp, assert_close, assert_close_out, dev, host, state_close

pytestmark = pytest.mark.gpu


def _hist(rng, B, D, W, dtype):
    h = rng.standard_normal((B, D, W - 1)).astype(np.float32)
    return synth.round_bf16(h) if dtype == "bf16" else h


def _piece(inp, a, b):
    out = dict(inp)
    for k in ("u", "delta", "z", "B", "C"):
        out[k] = np.ascontiguousarray(inp[k][..., a:b])
    return out


def _gpu(inp, dtype, *, conv=True, h0=None, hist=None, chunks=0, tail=True):
    t = lambda k: dev(inp[k], dtype)
    f = lambda k: dev(inp[k])
    res = ssm.ssm_selective_scan_fwd(
        t("u"), t("delta"), f("A"), t("B"), t("C"), f("D"), t("z"), f("delta_bias"), True, False,
        f("conv_w") if conv else None, f("conv_b") if conv else None, return_final_state=True,
        num_chunks=chunks, initial_state=None if h0 is None else dev(h0),
        conv_history=None if hist is None else dev(hist, dtype),
        return_conv_state=conv and tail)
    torch.cuda.synchronize()
    return res


def _oracle(inp, *, conv=True, h0=None, hist=None):
    return oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                 inp["z"], inp["delta_bias"], True, False,
                                 inp["conv_w"] if conv else None, inp["conv_b"] if conv else None,
                                 h0=h0, return_final_state=True, conv_hist=hist)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("conv", [True, False])
@pytest.mark.parametrize("chunks", [0, 3])
@pytest.mark.parametrize("shape", [(2, 40, 300, 16), (1, 33, 70, 5)], ids=str)
def test_initial_state_and_history_match_oracle(dtype, conv, chunks, shape):
    B, D, L, N = shape
    rng = np.random.default_rng(40)
    inp = synth.scan_inputs(B, D, L, N, dtype, conv_width=4 if conv else 0, seed=41)
    h0 = rng.standard_normal((B, D, N)).astype(np.float32)
    hist = _hist(rng, B, D, 4, dtype) if conv else None
    res = _gpu(inp, dtype, conv=conv, h0=h0, hist=hist, chunks=chunks)
    yo, ho = _oracle(inp, conv=conv, h0=h0, hist=hist)
    assert_close_out(host(res[0]), yo, dtype, "y")
    state_close(host(res[1]), ho, "final state")
    if conv:
        np.testing.assert_array_equal(host(res[2]), oracle.conv_tail(inp["u"], 4, hist))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("cuts", [(1,), (2,), (3,), (40,), (64,), (2, 3), (1, 2, 97), (130, 131)],
                         ids=str)
def test_prompt_in_pieces_matches_one_piece(dtype, cuts):
    """Each piece starts from the previous piece's final state and conv state (its last
    W-1 inputs); pieces shorter than W-1 make the history span several pieces."""
    B, D, L, N = 2, 40, 200, 16
    inp = synth.scan_inputs(B, D, L, N, dtype, conv_width=4, seed=42)
    y1, h1, _ = _gpu(inp, dtype)
    yo, ho = _oracle(inp)
    bounds = [0, *cuts, L]
    ys, st, hist = [], None, None
    for a, b in zip(bounds[:-1], bounds[1:]):
        yp, st, cs = _gpu(_piece(inp, a, b), dtype, h0=None if st is None else host(st),
                          hist=None if hist is None else host(hist))
        hist = cs[..., 1:].contiguous()
        ys.append(host(yp))
    y = np.concatenate(ys, axis=-1)
    assert_close_out(y, yo, dtype, "pieces vs oracle")
    state_close(host(st), ho, "final state")
    if dtype == "bf16":
        assert_bf16_ulp(y, host(y1), "pieces vs one piece")
    else:
        assert_close(y, host(y1), dtype, "pieces vs one piece")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_continues_a_gpu_scan(dtype):
    B, D, L, N, k = 2, 64, 48, 16, 31
    inp = synth.scan_inputs(B, D, L, N, dtype, conv_width=4, seed=43)
    yo, ho = _oracle(inp)
    _, st, cs = _gpu(_piece(inp, 0, k), dtype)
    t = lambda key, s: dev(np.ascontiguousarray(inp[key][..., s]), dtype)
    f = lambda key: dev(inp[key])
    for s in range(k, L):
        y = ssm.ssm_selective_state_update(st, cs, t("u", s), t("delta", s), f("A"), t("B", s),
                                           t("C", s), f("D"), t("z", s), f("delta_bias"), True,
                                           f("conv_w"), f("conv_b"))
        torch.cuda.synchronize()
        assert_close_out(host(y), yo[..., s], dtype, f"token {s}")
    state_close(host(st), ho, "state")


def test_history_plain_path_matches_tma(monkeypatch):
    """The TMA path patches the history into the landed halo; the plain-load path reads
    it while loading. Both must agree bit for bit."""
    B, D, L, N = 2, 40, 200, 16
    rng = np.random.default_rng(44)
    inp = synth.scan_inputs(B, D, L, N, "bf16", conv_width=4, seed=45)
    h0 = rng.standard_normal((B, D, N)).astype(np.float32)
    hist = _hist(rng, B, D, 4, "bf16")
    a = _gpu(inp, "bf16", h0=h0, hist=hist)
    monkeypatch.setenv("SSM_NO_TMA", "1")
    b = _gpu(inp, "bf16", h0=h0, hist=hist)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("L", [0, 1, 2])
def test_short_and_empty_sequences(L):
    """L = 0: the final state is the initial state and the conv state is the history;
    L < W - 1: the conv state mixes history and input."""
    B, D, N = 1, 32, 16
    rng = np.random.default_rng(46)
    inp = synth.scan_inputs(B, D, max(L, 1), N, "f32", conv_width=4, seed=47)
    if L == 0:
        inp = _piece(inp, 0, 0)
    h0 = rng.standard_normal((B, D, N)).astype(np.float32)
    hist = _hist(rng, B, D, 4, "f32")
    y, h, cs = _gpu(inp, "f32", h0=h0, hist=hist)
    np.testing.assert_array_equal(host(cs), oracle.conv_tail(inp["u"], 4, hist))
    if L == 0:
        np.testing.assert_array_equal(host(h), h0)
    else:
        yo, ho = _oracle(inp, h0=h0, hist=hist)
        assert_close_out(host(y), yo, "f32", "y")
        state_close(host(h), ho, "final state")


def test_state_updated_in_place():
    """final_state may be the initial_state buffer itself (one pass)."""
    B, D, L, N = 2, 40, 100, 16
    rng = np.random.default_rng(48)
    inp = synth.scan_inputs(B, D, L, N, "bf16", conv_width=4, seed=49)
    h0 = rng.standard_normal((B, D, N)).astype(np.float32)
    st = dev(h0)
    t = lambda k: dev(inp[k], "bf16")
    f = lambda k: dev(inp[k])
    ssm.ssm_selective_scan_fwd(t("u"), t("delta"), f("A"), t("B"), t("C"), f("D"), t("z"),
                               f("delta_bias"), True, False, f("conv_w"), f("conv_b"),
                               initial_state=st, final_state=st)
    torch.cuda.synchronize()
    _, ho = _oracle(inp, h0=h0)
    state_close(host(st), ho, "state")
