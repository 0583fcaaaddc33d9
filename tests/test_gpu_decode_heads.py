"""GPU parity of the decode step with d_state up to 128 and with A one scalar per head
(ssm_selective_state_update_ex, reached through the binding when A is 1-D or d_state is
above 16) against the CPU oracle, over several successive steps: ragged row counts,
d_state not a multiple of 4, both dtypes, with and without the conv and the gate; the
streaming kernel (d_state 32, 64, 128 in whole channel groups) over conv widths, short and
long per-CTA tile ranges and ranges that cross channel groups, beside the plain kernel;
and decode steps against the scan of the same sequence on the GPU."""
import os

import numpy as np
import pytest
import torch

import oracle
import mamba_selective_scan_sm_b200 as ssm
from mamba_selective_scan_sm_b200 import synth
from tests.gpu_helpers import assert_close_out, dev, host, state_close

pytestmark = pytest.mark.gpu


def _gpu(inp, dtype, steps, conv, gate):
    st = dev(inp["state"])
    cs = dev(inp["conv_state"], dtype)
    ys = []
    for s in range(steps):
        ys.append(ssm.ssm_selective_state_update(
            st, cs, dev(inp["x"][s], dtype), dev(inp["dt"][s], dtype), dev(inp["A"]),
            dev(inp["B"][s], dtype), dev(inp["C"][s], dtype), dev(inp["D"]),
            dev(inp["z"][s], dtype) if gate else None, dev(inp["dt_bias"]), True,
            dev(inp["conv_w"]) if conv else None, dev(inp["conv_b"]) if conv else None))
    torch.cuda.synchronize()
    return [host(y) for y in ys], host(st), host(cs)


def _ref(inp, steps, conv, gate):
    st, cs = inp["state"].astype(np.float64), inp["conv_state"].astype(np.float64)
    ys = []
    for s in range(steps):
        y, st, cs2 = oracle.state_update(st, cs if conv else None, inp["x"][s], inp["dt"][s],
                                         inp["A"], inp["B"][s], inp["C"][s], inp["D"],
                                         inp["z"][s] if gate else None, inp["dt_bias"], True,
                                         inp["conv_w"] if conv else None,
                                         inp["conv_b"] if conv else None)
        if conv:
            cs = cs2
        ys.append(y)
    return ys, st, cs


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,heads", [(16, 4), (32, 0), (64, 4), (100, 0), (128, 4), (128, 0),
                                     (7, 4)])
@pytest.mark.parametrize("conv,gate", [(True, True), (False, False)])
def test_decode_large_state_and_heads(dtype, N, heads, conv, gate):
    B, D, steps = 3, 44, 4                            # 132 rows: a partial warp of rows
    inp = synth.decode_inputs(B, D, N, steps, 4, dtype, seed=97, a_heads=heads)
    yg, sg, cg = _gpu(inp, dtype, steps, conv, gate)
    yo, so, co = _ref(inp, steps, conv, gate)
    for s in range(steps):
        assert_close_out(yg[s], yo[s], dtype, f"y step {s}")
    state_close(sg, so, "state")
    if conv:
        np.testing.assert_array_equal(cg, co)        # the conv state holds copied inputs


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,heads", [(128, 6), (64, 0)])
def test_decode_steps_equal_scan_on_gpu(dtype, N, heads):
    """L decode steps from a zero state and zero conv history give the scan's outputs and
    final state (both on the GPU)."""
    B, D, L = 2, 48, 40
    inp = synth.scan_inputs(B, D, L, N, dtype, conv_width=4, seed=98, a_heads=heads)
    t = lambda k: dev(inp[k], dtype)
    f = lambda k: dev(inp[k])
    y, h = ssm.ssm_selective_scan_fwd(t("u"), t("delta"), f("A"), t("B"), t("C"), f("D"), t("z"),
                                      f("delta_bias"), True, False, f("conv_w"), f("conv_b"),
                                      return_final_state=True)
    st = torch.zeros(B, D, N, device="cuda")
    cs = torch.zeros(B, D, 4, device="cuda", dtype=t("u").dtype)
    ys = []
    for s in range(L):
        ys.append(ssm.ssm_selective_state_update(
            st, cs, t("u")[..., s].contiguous(), t("delta")[..., s].contiguous(), f("A"),
            t("B")[..., s].contiguous(), t("C")[..., s].contiguous(), f("D"),
            t("z")[..., s].contiguous(), f("delta_bias"), True, f("conv_w"), f("conv_b")))
    torch.cuda.synchronize()
    yd = np.stack([host(v) for v in ys], axis=-1)
    assert_close_out(yd, host(y), dtype, "decode vs scan", ulp=False)
    state_close(host(st), host(h), "decode vs scan state")


def _check(inp, dtype, steps, conv, gate):
    # a nonzero conv bias, so that a dropped or misplaced bias shows
    inp["conv_b"] = np.random.default_rng(7).normal(0, 0.5, inp["conv_b"].shape).astype(np.float32)
    yg, sg, cg = _gpu(inp, dtype, steps, conv, gate)
    yo, so, co = _ref(inp, steps, conv, gate)
    for s in range(steps):
        assert_close_out(yg[s], yo[s], dtype, f"y step {s}")
    state_close(sg, so, "state")
    if conv:
        np.testing.assert_array_equal(cg, co)


# (d_state, heads, dim): dim a whole number of 4096 / d_state channel groups
STREAM_SHAPES = [(128, 4, 96), (128, 0, 64), (64, 3, 192), (64, 0, 128), (32, 2, 256),
                 (32, 0, 128)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,heads,D", STREAM_SHAPES)
@pytest.mark.parametrize("width,gate", [(4, True), (3, False), (2, True), (1, False), (0, True)])
@pytest.mark.parametrize("kernel", ["", "plain"])
def test_streaming_decode_shapes(dtype, N, heads, D, width, gate, kernel, monkeypatch):
    """The streaming kernel (default for these shapes) and the plain one, against the
    oracle: one tile per CTA (B * D / group tiles below one wave)."""
    monkeypatch.setenv("SSM_DECODE_KERNEL", kernel)
    inp = synth.decode_inputs(5, D, N, 3, max(width, 1), dtype, seed=101, a_heads=heads)
    _check(inp, dtype, 3, width > 0, gate)


@pytest.mark.parametrize("dtype,N,heads,B,D", [("bf16", 128, 4, 1000, 96), ("f32", 128, 0, 700, 64),
                                              ("f32", 32, 2, 600, 256), ("bf16", 64, 0, 450, 192)])
def test_streaming_decode_long_ranges(dtype, N, heads, B, D):
    """More tiles than one wave of CTAs: each CTA walks a range of several tiles through
    the copy ring, and ranges cross from one channel group into the next."""
    assert os.environ.get("SSM_DECODE_KERNEL", "") in ("", "stream")
    inp = synth.decode_inputs(B, D, N, 2, 4, dtype, seed=102, a_heads=heads)
    _check(inp, dtype, 2, True, True)
