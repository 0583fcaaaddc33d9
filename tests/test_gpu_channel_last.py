"""GPU parity of channel-last activations: u, delta, z, out as (batch, seqlen, dim) and
B, C as (batch, seqlen, dstate), dense or as views with a position stride (the x and z
halves of an in_proj output, the B and C columns of an x_proj output). The layout only
moves data: results equal the (batch, dim, seqlen) call bit for bit, and the oracle on
the transposed inputs."""
import numpy as np
import pytest
import torch

import oracle
import mamba_selective_scan_sm_b200 as ssm
from mamba_selective_scan_sm_b200 import synth
from tests.gpu_helpers import assert_close_out, dev, host, state_close

pytestmark = pytest.mark.gpu

ACT = ("u", "delta", "z", "B", "C")


def _tensors(inp, dtype):
    t = {k: dev(inp[k], dtype) for k in ACT}
    f = {k: dev(inp[k]) for k in ("A", "D", "delta_bias", "conv_w", "conv_b", "A_rev", "D_rev",
                                  "delta_bias_rev") if inp.get(k) is not None}
    return t, f


def _call(t, f, *, cl, conv, reverse=False, bidir=False, chunks=0, **kw):
    g = (lambda k: t[k].transpose(1, 2).contiguous()) if cl else (lambda k: t[k])
    return ssm.ssm_selective_scan_fwd(
        g("u"), g("delta"), f["A"], g("B"), g("C"), f["D"], g("z"), f["delta_bias"], True,
        reverse, f["conv_w"] if conv else None, f["conv_b"] if conv else None,
        f.get("A_rev") if bidir else None, f.get("D_rev") if bidir else None,
        f.get("delta_bias_rev") if bidir else None, return_final_state=True,
        num_chunks=chunks, channel_last=cl, **kw)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("conv", [True, False])
@pytest.mark.parametrize("mode", ["fwd", "rev", "bidir"])
@pytest.mark.parametrize("chunks", [0, 1, 3])
@pytest.mark.parametrize("shape", [(2, 40, 200, 16), (1, 33, 333, 16), (2, 24, 96, 5),
                                   (1, 16, 70, 3)], ids=str)
def test_channel_last_equals_standard_layout(dtype, conv, mode, chunks, shape):
    B, D, L, N = shape
    if mode == "bidir" and chunks == 3:
        pytest.skip("the bidirectional sum runs as a single pass")
    inp = synth.scan_inputs(B, D, L, N, dtype, conv_width=4 if conv else 0,
                            bidirectional=mode == "bidir", seed=70)
    t, f = _tensors(inp, dtype)
    kw = dict(conv=conv, reverse=mode == "rev", bidir=mode == "bidir", chunks=chunks)
    a = _call(t, f, cl=False, **kw)
    b = _call(t, f, cl=True, **kw)
    torch.cuda.synchronize()
    assert torch.equal(b[0].transpose(1, 2), a[0])
    for x, y in zip(a[1:], b[1:]):
        assert torch.equal(x, y)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dt_rank", [48, 47])
def test_views_into_projection_outputs(dtype, dt_rank):
    """x, z: halves of one (batch, seqlen, 2*dim) tensor; B, C: columns of one
    (batch, seqlen, dt_rank + 2*dstate) tensor. dt_rank 48 keeps every stride a multiple
    of 16 bytes (TMA); 47 does not (plain loads)."""
    B, D, L, N = 2, 64, 160, 16
    inp = synth.scan_inputs(B, D, L, N, dtype, conv_width=4, seed=71)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    xz = torch.empty(B, L, 2 * D, dtype=tdt, device="cuda")
    xz[..., :D] = dev(inp["u"], dtype).transpose(1, 2)
    xz[..., D:] = dev(inp["z"], dtype).transpose(1, 2)
    xdbl = torch.zeros(B, L, dt_rank + 2 * N, dtype=tdt, device="cuda")
    xdbl[..., dt_rank:dt_rank + N] = dev(inp["B"], dtype).transpose(1, 2)
    xdbl[..., dt_rank + N:] = dev(inp["C"], dtype).transpose(1, 2)
    dt = dev(inp["delta"], dtype).transpose(1, 2).contiguous()
    y, h = ssm.ssm_selective_scan_fwd(
        xz[..., :D], dt, dev(inp["A"]), xdbl[..., dt_rank:dt_rank + N], xdbl[..., dt_rank + N:],
        dev(inp["D"]), xz[..., D:], dev(inp["delta_bias"]), True, False, dev(inp["conv_w"]),
        dev(inp["conv_b"]), return_final_state=True, channel_last=True)
    torch.cuda.synchronize()
    yo, ho = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                                   inp["z"], inp["delta_bias"], True, False, inp["conv_w"],
                                   inp["conv_b"], return_final_state=True)
    assert_close_out(host(y.transpose(1, 2)), yo, dtype, "y")
    state_close(host(h), ho, "final state")


def test_channel_last_plain_path_matches_tma(monkeypatch):
    inp = synth.scan_inputs(2, 40, 200, 16, "bf16", conv_width=4, seed=72)
    t, f = _tensors(inp, "bf16")
    a = _call(t, f, cl=True, conv=True)
    monkeypatch.setenv("SSM_NO_TMA", "1")
    b = _call(t, f, cl=True, conv=True)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_channel_last_packed_and_continued(dtype):
    """Channel-last with packed sequences, and with an initial state, conv history and
    the conv state handed on: equal to the standard layout."""
    inp = synth.scan_inputs(1, 40, 300, 16, dtype, conv_width=4, seed=73)
    t, f = _tensors(inp, dtype)
    starts = torch.tensor([0, 3, 100, 101, 300], dtype=torch.int32, device="cuda")
    a = _call(t, f, cl=False, conv=True, seq_starts=starts, return_conv_state=True)
    b = _call(t, f, cl=True, conv=True, seq_starts=starts, return_conv_state=True)
    torch.cuda.synchronize()
    assert torch.equal(b[0].transpose(1, 2), a[0])
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    rng = np.random.default_rng(74)
    h0 = dev(rng.standard_normal((1, 40, 16)).astype(np.float32))
    hist = dev(synth.round_bf16(rng.standard_normal((1, 40, 3)).astype(np.float32))
               if dtype == "bf16" else rng.standard_normal((1, 40, 3)).astype(np.float32), dtype)
    kw = dict(initial_state=h0, conv_history=hist, return_conv_state=True)
    a = _call(t, f, cl=False, conv=True, **kw)
    b = _call(t, f, cl=True, conv=True, **kw)
    torch.cuda.synchronize()
    assert torch.equal(b[0].transpose(1, 2), a[0])
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
