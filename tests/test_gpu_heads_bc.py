"""GPU parity of the scan with A as one scalar per head (every state of a head's
channels decays by exp(delta * A_h): one exp per channel and step), with time-invariant
B/C (fp32 (dim, dstate), fixed per channel), and with d_state 64 and 128, against the
CPU oracle element by element: several tiles, ragged seqlen, both dtypes, forward,
reverse and the bidirectional sum, the fused conv, final states, the two-pass carry,
channel-last activations and the plain-load path."""
import numpy as np
import pytest
import torch

import oracle
import mamba_selective_scan_sm_b200 as ssm
from mamba_selective_scan_sm_b200 import synth
from tests.gpu_helpers import assert_close_out, dev, host, state_close

pytestmark = pytest.mark.gpu


def _inputs(B, D, L, N, dtype, heads, shared, bidir=False, seed=90):
    return synth.scan_inputs(B, D, L, N, dtype, conv_width=4, bidirectional=bidir, seed=seed,
                             a_heads=heads, bc_shared=shared)


def _gpu(inp, dtype, *, mode="fwd", chunks=0, cl=False):
    shared = inp["B"].ndim == 2
    act = lambda k: dev(inp[k], dtype)
    par = lambda k: dev(inp[k]) if inp.get(k) is not None else None
    t = {k: act(k) for k in ("u", "delta", "z")}
    bc = {k: (par(k) if shared else act(k)) for k in ("B", "C")}
    if cl:
        t = {k: v.transpose(1, 2).contiguous() for k, v in t.items()}
        if not shared:
            bc = {k: v.transpose(1, 2).contiguous() for k, v in bc.items()}
    bidir = mode == "bidir"
    res = ssm.ssm_selective_scan_fwd(
        t["u"], t["delta"], par("A"), bc["B"], bc["C"], par("D"), t["z"], par("delta_bias"),
        True, mode == "rev", par("conv_w"), par("conv_b"), par("A_rev") if bidir else None,
        par("D_rev") if bidir else None, par("delta_bias_rev") if bidir else None,
        return_final_state=True, num_chunks=chunks, channel_last=cl)
    torch.cuda.synchronize()
    y = res[0].transpose(1, 2) if cl else res[0]
    return (host(y),) + tuple(host(r) for r in res[1:])


def _ref(inp, mode="fwd"):
    if mode == "bidir":
        return oracle.selective_scan_bidir(
            inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["z"],
            inp["delta_bias"], inp["A_rev"], inp["D_rev"], inp["delta_bias_rev"], True,
            inp["conv_w"], inp["conv_b"], return_final_state=True)
    return oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                 inp["z"], inp["delta_bias"], True, mode == "rev", inp["conv_w"],
                                 inp["conv_b"], return_final_state=True)


def _check(g, o, dtype, what):
    assert_close_out(g[0], o[0], dtype, what)
    for gs, os_ in zip(g[1:], o[1:]):
        state_close(gs, os_, what + " state")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [16, 64, 128])
@pytest.mark.parametrize("heads,shared", [(4, False), (0, True), (4, True), (0, False)])
@pytest.mark.parametrize("mode", ["fwd", "rev", "bidir"])
def test_heads_shared_bc_large_state(dtype, N, heads, shared, mode):
    if N == 16 and heads == 0 and not shared:
        pytest.skip("the per-state, input-dependent N = 16 scan is covered in test_gpu_scan")
    inp = _inputs(2, 48, 150, N, dtype, heads, shared, bidir=mode == "bidir")
    _check(_gpu(inp, dtype, mode=mode), _ref(inp, mode), dtype,
           f"N={N} heads={heads} shared={shared} {mode}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,heads,shared", [(128, 4, False), (64, 0, True), (16, 4, True)])
@pytest.mark.parametrize("chunks", [3, 8])
def test_two_pass_carry(dtype, N, heads, shared, chunks):
    inp = _inputs(1, 24, 700, N, dtype, heads, shared, seed=91)
    _check(_gpu(inp, dtype, chunks=chunks), _ref(inp), dtype, f"chunks={chunks}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,heads,shared", [(128, 4, False), (16, 4, True), (64, 0, False)])
@pytest.mark.parametrize("mode", ["fwd", "bidir"])
def test_channel_last_equals_standard_layout(dtype, N, heads, shared, mode):
    inp = _inputs(2, 40, 200, N, dtype, heads, shared, bidir=mode == "bidir", seed=92)
    a = _gpu(inp, dtype, mode=mode)
    b = _gpu(inp, dtype, mode=mode, cl=True)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


@pytest.mark.parametrize("N,heads,shared", [(128, 4, False), (16, 4, True)])
def test_plain_loads_match_tma(monkeypatch, N, heads, shared):
    inp = _inputs(2, 40, 256, N, "bf16", heads, shared, seed=93)
    a = _gpu(inp, "bf16")
    monkeypatch.setenv("SSM_NO_TMA", "1")
    b = _gpu(inp, "bf16")
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_one_head_spans_all_channels():
    """a_heads = 1: every channel shares one decay."""
    inp = _inputs(1, 32, 100, 64, "f32", 1, False, seed=94)
    _check(_gpu(inp, "f32"), _ref(inp), "f32", "one head")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("per_lane", ["1", "2"])
@pytest.mark.parametrize("mode", ["fwd", "bidir"])
def test_heads_channels_per_lane(monkeypatch, dtype, N, per_lane, mode):
    """d_state 64 / 128 with A per head: one or two channels per lane (the default, which
    shares each lane's B/C loads between its channels), on a ragged channel count."""
    monkeypatch.setenv("SSM_CHANNELS_PER_LANE", per_lane)
    inp = _inputs(2, 40, 150, N, dtype, 4, False, bidir=mode == "bidir", seed=95)
    _check(_gpu(inp, dtype, mode=mode), _ref(inp, mode), dtype, f"per_lane={per_lane}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("scan_warps", ["4", "8"])
def test_heads_large_state_cta_sizes(monkeypatch, dtype, scan_warps):
    """d_state 128, A per head, two channels per lane: CTAs of 4 scan warps (16 channels)
    and of 8 (32 channels, the default), with a channel count that leaves a partial CTA."""
    monkeypatch.setenv("SSM_SCAN_WARPS", scan_warps)
    inp = _inputs(2, 72, 130, 128, dtype, 6, False, seed=96)
    _check(_gpu(inp, dtype, chunks=2), _ref(inp), dtype, f"scan warps {scan_warps}")
