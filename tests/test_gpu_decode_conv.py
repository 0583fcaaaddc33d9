"""GPU parity of ssm_selective_state_update (decode) and ssm_causal_conv1d_fwd
against the CPU oracle, plus the decode/scan consistency on the GPU."""
import numpy as np
import pytest
import torch

import oracle
import mamba_selective_scan_sm_b200 as ssm
from mamba_selective_scan_sm_b200 import synth
from tests.gpu_helpers import assert_bf16_ulp, assert_close, assert_close_out, dev, host, state_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", [(2, 5, 40, 16), (1, 3, 333, 16), (2, 7, 64, 4), (1, 4, 1, 16)],
                         ids=str)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("width", [2, 3, 4])
@pytest.mark.parametrize("silu", [True, False])
def test_conv_matches_oracle(shape, dtype, width, silu):
    B, D, L, _ = shape
    rng = np.random.default_rng(21)
    x = rng.standard_normal((B, D, L)).astype(np.float32)
    if dtype == "bf16":
        x = synth.round_bf16(x)
    w = (0.5 * rng.standard_normal((D, width))).astype(np.float32)
    b = rng.standard_normal(D).astype(np.float32)
    y = ssm.ssm_causal_conv1d_fwd(dev(x, dtype), dev(w), dev(b), silu)
    torch.cuda.synchronize()
    assert_close_out(host(y), oracle.causal_conv1d(x, w, b, silu), dtype, "conv")


def test_conv_aligned_long_rows():
    x = synth.round_bf16(np.random.default_rng(22).standard_normal((4, 64, 4096)).astype(np.float32))
    w = (0.5 * np.random.default_rng(23).standard_normal((64, 4))).astype(np.float32)
    y = ssm.ssm_causal_conv1d_fwd(dev(x, "bf16"), dev(w), None, True)
    torch.cuda.synchronize()
    assert_close_out(host(y), oracle.causal_conv1d(x, w, None, True), "bf16", "conv")


def _decode_gpu(inp, dtype, steps, conv=True, gate=True, skip=True):
    st = dev(inp["state"])
    cs = dev(inp["conv_state"], dtype)
    ys = []
    for s in range(steps):
        ys.append(ssm.ssm_selective_state_update(
            st, cs, dev(inp["x"][s], dtype), dev(inp["dt"][s], dtype), dev(inp["A"]),
            dev(inp["B"][s], dtype), dev(inp["C"][s], dtype), dev(inp["D"]) if skip else None,
            dev(inp["z"][s], dtype) if gate else None, dev(inp["dt_bias"]), True,
            dev(inp["conv_w"]) if conv else None, dev(inp["conv_b"]) if conv else None))
    torch.cuda.synchronize()
    return [host(y) for y in ys], host(st), host(cs)


def _decode_oracle(inp, steps, conv=True, gate=True, skip=True):
    st, cs = inp["state"].astype(np.float64), inp["conv_state"].astype(np.float64)
    ys = []
    for s in range(steps):
        y, st, cs2 = oracle.state_update(st, cs if conv else None, inp["x"][s], inp["dt"][s],
                                         inp["A"], inp["B"][s], inp["C"][s],
                                         inp["D"] if skip else None, inp["z"][s] if gate else None,
                                         inp["dt_bias"], True, inp["conv_w"] if conv else None,
                                         inp["conv_b"] if conv else None)
        if conv:
            cs = cs2
        ys.append(y)
    return ys, st, cs


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dstate", [16, 5])
@pytest.mark.parametrize("opts", [dict(), dict(conv=False), dict(gate=False, skip=False)],
                         ids=["full", "no-conv", "no-z-no-D"])
def test_decode_matches_oracle(dtype, dstate, opts):
    B, D, steps = 3, 37, 8
    inp = synth.decode_inputs(B, D, dstate, steps, 4, dtype, seed=24)
    yg, sg, cg = _decode_gpu(inp, dtype, steps, **opts)
    yo, so, co = _decode_oracle(inp, steps, **opts)
    for s in range(steps):
        assert_close_out(yg[s], yo[s], dtype, f"y step {s}")
    state_close(sg, so, "state")
    if opts.get("conv", True):
        np.testing.assert_array_equal(cg, co)   # conv state holds copied inputs: exact


def test_decode_graph_capture_64_steps():
    """64 steps captured in one CUDA graph replay to the same result as eager calls."""
    B, D, N, steps = 4, 96, 16, 64
    inp = synth.decode_inputs(B, D, N, steps, 4, "bf16", seed=25)
    X = [dev(inp[k], "bf16") for k in ("x", "dt", "z", "B", "C")]
    A, Dv, db, cw, cb = (dev(inp[k]) for k in ("A", "D", "dt_bias", "conv_w", "conv_b"))
    outs = torch.empty(steps, B, D, dtype=torch.bfloat16, device="cuda")

    def run(st, cs):
        for s in range(steps):
            ssm.ssm_selective_state_update(st, cs, X[0][s], X[1][s], A, X[3][s], X[4][s], Dv,
                                           X[2][s], db, True, cw, cb, out=outs[s])

    st_e, cs_e = dev(inp["state"]), dev(inp["conv_state"], "bf16")
    run(st_e, cs_e)
    ref = outs.clone()
    st_g, cs_g = dev(inp["state"]), dev(inp["conv_state"], "bf16")
    st0, cs0 = st_g.clone(), cs_g.clone()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run(st_g, cs_g)                                 # warm-up outside capture
    torch.cuda.current_stream().wait_stream(s)
    st_g.copy_(st0), cs_g.copy_(cs0)
    with torch.cuda.graph(g):
        run(st_g, cs_g)
    st_g.copy_(st0), cs_g.copy_(cs0)
    outs.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(outs, ref)
    assert torch.equal(st_g, st_e) and torch.equal(cs_g, cs_e)
    yo, so, _ = _decode_oracle(inp, steps)
    for k in range(steps):
        assert_close_out(host(outs[k]), yo[k], "bf16", f"step {k}")
    state_close(host(st_g), so, "state")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_repeated_equals_scan_on_gpu(dtype):
    """L decode steps from a zero state and zero conv history reproduce the fused-conv scan
    (both on the GPU)."""
    B, D, L, N = 2, 40, 48, 16
    inp = synth.scan_inputs(B, D, L, N, dtype, conv_width=4, seed=26)
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
    yd = torch.stack(ys, -1)
    if dtype == "bf16":
        assert_bf16_ulp(host(yd), host(y), "decode^L vs scan")
    else:
        assert_close(host(yd), host(y), dtype, "decode^L vs scan")
    state_close(host(st), host(h), "state")


@pytest.mark.parametrize("kernel", ["stream", "bulk"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dstate", [16, 5])
@pytest.mark.parametrize("width", [4, 2, 3])
@pytest.mark.parametrize("opts", [dict(), dict(conv=False), dict(gate=False, skip=False)],
                         ids=["full", "no-conv", "no-z-no-D"])
def test_decode_fast_paths_match_oracle(monkeypatch, kernel, dtype, dstate, width, opts):
    """Channel counts a multiple of 64 with 16-byte aligned bases take the streaming
    kernel (dstate 16) or the bulk-copy kernel; other dstates fall back to plain loads."""
    monkeypatch.setenv("SSM_DECODE_KERNEL", kernel)
    B, D, steps = 2, 128, 6
    inp = synth.decode_inputs(B, D, dstate, steps, width, dtype, seed=27)
    yg, sg, cg = _decode_gpu(inp, dtype, steps, **opts)
    yo, so, co = _decode_oracle(inp, steps, **opts)
    for s in range(steps):
        assert_close_out(yg[s], yo[s], dtype, f"y step {s}")
    state_close(sg, so, "state")
    if opts.get("conv", True):
        np.testing.assert_array_equal(cg, co)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_stream_many_batch_rows_per_cta(dtype):
    """Enough batch rows that each CTA of the streaming kernel walks more tiles than its
    copy ring has stages (200 rows in ranges of 14), with a ragged last range."""
    B, D, steps = 200, 5120, 2
    inp = synth.decode_inputs(B, D, 16, steps, 4, dtype, seed=29)
    yg, sg, cg = _decode_gpu(inp, dtype, steps)
    yo, so, co = _decode_oracle(inp, steps)
    for s in range(steps):
        assert_close_out(yg[s], yo[s], dtype, f"y step {s}")
    state_close(sg, so, "state")
    np.testing.assert_array_equal(cg, co)


def test_decode_kernels_agree(monkeypatch):
    """Streaming, bulk-copy and plain-load kernels give the same steps."""
    B, D, steps = 3, 256, 4
    inp = synth.decode_inputs(B, D, 16, steps, 4, "bf16", seed=28)
    res = {}
    for kernel in ("stream", "bulk", "plain"):
        monkeypatch.setenv("SSM_DECODE_KERNEL", kernel)
        res[kernel] = _decode_gpu(inp, "bf16", steps)
    yp, sp, cp = res["plain"]
    for kernel in ("stream", "bulk"):
        yk, sk, ck = res[kernel]
        for s in range(steps):
            assert_bf16_ulp(yk[s], yp[s], f"{kernel} step {s}")
        state_close(sk, sp, f"{kernel} state")
        np.testing.assert_array_equal(ck, cp)
