"""Parity at the full workload sizes, in the launch configuration the benchmark
times (automatic variant and chunk choice), on sampled channels: every channel's
scan is independent, so the oracle computes a sample of (batch, channel) rows in
full and the GPU's rows are compared element by element."""
import numpy as np
import pytest
import torch

import oracle
import mamba_selective_scan_sm_b200 as ssm
from mamba_selective_scan_sm_b200 import synth
from tests.gpu_helpers import assert_close_out, dev, host, state_close

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _sample(batch, dim, n, seed=0):
    rng = np.random.default_rng(seed)
    picks = {(0, 0), (batch - 1, dim - 1), (0, dim - 1), (batch - 1, 0)}
    while len(picks) < n:
        picks.add((int(rng.integers(batch)), int(rng.integers(dim))))
    return sorted(picks)


def _gpu_scan(inp, w, **kw):
    t = lambda k: dev(inp[k], w.dtype)
    f = lambda k: dev(inp[k]) if inp.get(k) is not None else None
    conv = w.conv_width > 0
    res = ssm.ssm_selective_scan_fwd(
        t("u"), t("delta"), f("A"), t("B"), t("C"), f("D"), t("z"), f("delta_bias"), True,
        False, f("conv_w") if conv else None, f("conv_b") if conv else None,
        f("A_rev") if w.bidirectional else None, f("D_rev") if w.bidirectional else None,
        f("delta_bias_rev") if w.bidirectional else None, return_final_state=True, **kw)
    torch.cuda.synchronize()
    return res


def _check(w, res, inp, chans):
    ref = oracle.scan_channels(inp, chans, conv=w.conv_width > 0, final_state=True,
                               bidirectional=w.bidirectional)
    y = res[0]
    rows = torch.tensor([b * w.dim + d for b, d in chans], device="cuda")
    yg = host(y.reshape(-1, w.seqlen)[rows])
    assert_close_out(yg, ref[0], w.dtype, w.name)
    hg = host(res[1].reshape(-1, res[1].shape[-1])[rows])
    state_close(hg, ref[1], "final state")
    if w.bidirectional:
        hr = host(res[2].reshape(-1, res[2].shape[-1])[rows])
        state_close(hr, ref[2], "reverse final state")


@pytest.mark.parametrize("key", ["m130", "bidir", "tiny"])
def test_fullsize_scan(key):
    w = synth.WORKLOADS[key]
    inp = synth.scan_inputs(w.batch, w.dim, w.seqlen, w.dstate, w.dtype, w.conv_width,
                            w.bidirectional, seed=0)
    res = _gpu_scan(inp, w)
    chans = _sample(w.batch, w.dim, 24 if key != "tiny" else 64)
    _check(w, res, inp, chans)


def test_fullsize_channel_last_block_layout():
    """The Mamba-130M layer in the block's own layout (x, z halves of the in_proj output,
    B, C columns of the x_proj output), as the benchmark times it: sampled channels
    against the oracle, and every element equal to the (batch, dim, seqlen) call."""
    w = synth.WORKLOADS["m130_cl"]
    B, D, L, N, R = w.batch, w.dim, w.seqlen, w.dstate, w.extra["dt_rank"]
    inp = synth.scan_inputs(B, D, L, N, w.dtype, w.conv_width, False, seed=0)
    cl = lambda k: dev(inp[k], w.dtype).transpose(1, 2)
    xz = torch.cat([cl("u"), cl("z")], dim=2).contiguous()
    xdbl = torch.zeros(B, L, R + 2 * N, dtype=xz.dtype, device="cuda")
    xdbl[..., R:R + N] = cl("B")
    xdbl[..., R + N:] = cl("C")
    f = lambda k: dev(inp[k])
    y, h = ssm.ssm_selective_scan_fwd(
        xz[..., :D], cl("delta").contiguous(), f("A"), xdbl[..., R:R + N], xdbl[..., R + N:],
        f("D"), xz[..., D:], f("delta_bias"), True, False, f("conv_w"), f("conv_b"),
        return_final_state=True, channel_last=True)
    torch.cuda.synchronize()
    res = (y.transpose(1, 2).contiguous(), h)
    _check(w, res, inp, _sample(B, D, 24))
    ref = _gpu_scan(inp, w)
    assert torch.equal(res[0], ref[0]) and torch.equal(res[1], ref[1])


@pytest.mark.parametrize("chunks", [0, 8])
def test_fullsize_long_sequence(chunks):
    """65536 steps: the automatic choice and an explicit 8-chunk two-pass carry."""
    w = synth.WORKLOADS["long"]
    inp = synth.scan_inputs(w.batch, w.dim, w.seqlen, w.dstate, w.dtype, 0, False, seed=0)
    res = _gpu_scan(inp, w, num_chunks=chunks)
    _check(w, res, inp, _sample(w.batch, w.dim, 8))


def test_fullsize_decode_h128_64_steps():
    """The d_state 128, A-per-head decode workload at full size (the streaming kernel, one
    wave of CTAs walking 16 KB state tiles), 64 steps, against the oracle on sampled rows."""
    w = synth.WORKLOADS["decode_h128"]
    B, D, N, steps, H = w.batch, w.dim, w.dstate, w.steps, w.extra["a_heads"]
    inp = synth.decode_inputs(B, D, N, steps, 4, "bf16", seed=0, a_heads=H)
    st = dev(inp["state"])
    cs = dev(inp["conv_state"], "bf16")
    X = {k: dev(inp[k], "bf16") for k in ("x", "dt", "z", "B", "C")}
    P = {k: dev(inp[k]) for k in ("A", "D", "dt_bias", "conv_w", "conv_b")}
    outs = torch.empty(steps, B, D, dtype=torch.bfloat16, device="cuda")
    for s in range(steps):
        ssm.ssm_selective_state_update(st, cs, X["x"][s], X["dt"][s], P["A"], X["B"][s],
                                       X["C"][s], P["D"], X["z"][s], P["dt_bias"], True,
                                       P["conv_w"], P["conv_b"], out=outs[s])
    torch.cuda.synchronize()
    og, sg = host(outs), host(st)
    hd = D // H
    for b, d in _sample(B, D, 16):
        so = inp["state"][b:b + 1, d:d + 1].astype(np.float64)
        co = inp["conv_state"][b:b + 1, d:d + 1].astype(np.float64)
        a_d = inp["A"][d // hd:d // hd + 1]          # the channel's head: one head of one channel
        yo = []
        for s in range(steps):
            sl = lambda k: inp[k][s, b:b + 1, d:d + 1]
            y, so, co = oracle.state_update(
                so, co, sl("x"), sl("dt"), a_d, inp["B"][s, b:b + 1], inp["C"][s, b:b + 1],
                inp["D"][d:d + 1], sl("z"), inp["dt_bias"][d:d + 1], True,
                inp["conv_w"][d:d + 1], inp["conv_b"][d:d + 1])
            yo.append(y[0, 0])
        assert_close_out(og[:, b, d], np.array(yo), "bf16", f"decode channel {(b, d)}")
        state_close(sg[b, d], so[0, 0], "state")


def test_fullsize_decode_64_steps():
    w = synth.WORKLOADS["decode"]
    B, D, N, steps = w.batch, w.dim, w.dstate, w.steps
    inp = synth.decode_inputs(B, D, N, steps, 4, "bf16", seed=0)
    st = dev(inp["state"])
    cs = dev(inp["conv_state"], "bf16")
    X = {k: dev(inp[k], "bf16") for k in ("x", "dt", "z", "B", "C")}
    P = {k: dev(inp[k]) for k in ("A", "D", "dt_bias", "conv_w", "conv_b")}
    outs = torch.empty(steps, B, D, dtype=torch.bfloat16, device="cuda")
    for s in range(steps):
        ssm.ssm_selective_state_update(st, cs, X["x"][s], X["dt"][s], P["A"], X["B"][s],
                                       X["C"][s], P["D"], X["z"][s], P["dt_bias"], True,
                                       P["conv_w"], P["conv_b"], out=outs[s])
    torch.cuda.synchronize()
    chans = _sample(B, D, 32)
    og = host(outs)
    sg = host(st)
    for b, d in chans:
        so = inp["state"][b:b + 1, d:d + 1].astype(np.float64)
        co = inp["conv_state"][b:b + 1, d:d + 1].astype(np.float64)
        yo = []
        for s in range(steps):
            sl = lambda k: inp[k][s, b:b + 1, d:d + 1]
            y, so, co = oracle.state_update(
                so, co, sl("x"), sl("dt"), inp["A"][d:d + 1], inp["B"][s, b:b + 1],
                inp["C"][s, b:b + 1], inp["D"][d:d + 1], sl("z"), inp["dt_bias"][d:d + 1], True,
                inp["conv_w"][d:d + 1], inp["conv_b"][d:d + 1])
            yo.append(y[0, 0])
        assert_close_out(og[:, b, d], np.array(yo), "bf16", f"decode channel {(b, d)}")
        state_close(sg[b, d], so[0, 0], "state")
