"""ssm_selective_scan_fwd_noalloc against ssm_selective_scan_fwd, through the C ABI.

The no-allocation entry point serves callers that cannot call cudaMalloc (they
can only pass buffers they already own): its scratch is a fixed array inside the
library. Here it must give the same results as the regular entry point given a
caller-allocated workspace, on two calls in a row, and it must refuse a call whose
scratch would not fit, without launching anything. Before the compared calls, one
call on the same shape with other inputs fills the shared scratch with unrelated
values, so a kernel that read scratch it had not written would show it.

The file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import mamba_selective_scan_sm_b200 as ssm
from mamba_selective_scan_sm_b200 import _abi, synth
from tests.gpu_helpers import assert_bf16_ulp, assert_close, dev, host, state_close

pytestmark = pytest.mark.gpu


def _args(inp, dtype, *, conv, bidir, chunks, out, fs, fsr):
    t = {k: dev(inp[k], dtype) for k in ("u", "delta", "z", "B", "C")}
    f = {k: dev(inp[k]) for k in ("A", "D", "delta_bias", "conv_w", "conv_b", "A_rev", "D_rev",
                                   "delta_bias_rev") if inp.get(k) is not None}
    a = _abi.ScanArgs()
    a.dtype = _abi.SSM_BF16 if dtype == "bf16" else _abi.SSM_F32
    a.batch, a.dim, a.seqlen = t["u"].shape
    a.dstate = f["A"].shape[1]
    a.u, a.delta, a.z, a.B, a.C = (t[k].data_ptr() for k in ("u", "delta", "z", "B", "C"))
    a.A, a.D, a.delta_bias = f["A"].data_ptr(), f["D"].data_ptr(), f["delta_bias"].data_ptr()
    a.delta_softplus = 1
    if conv:
        a.conv_weight, a.conv_bias, a.conv_width = f["conv_w"].data_ptr(), f["conv_b"].data_ptr(), 4
    if bidir:
        a.A_rev, a.D_rev = f["A_rev"].data_ptr(), f["D_rev"].data_ptr()
        a.delta_bias_rev = f["delta_bias_rev"].data_ptr()
        a.final_state_rev = fsr.data_ptr()
    a.out, a.final_state = out.data_ptr(), fs.data_ptr()
    a.num_chunks = chunks
    return a, (t, f)     # keep the tensors alive while the struct points at them


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


CASES = [
    dict(shape=(1, 40, 1000, 16), dtype="bf16", conv=True, bidir=False, chunks=4),  # summaries
    dict(shape=(2, 40, 300, 16), dtype="bf16", conv=False, bidir=True, chunks=0),   # fp32 partial
    dict(shape=(1, 33, 333, 16), dtype="f32", conv=True, bidir=False, chunks=3),
    dict(shape=(2, 24, 200, 16), dtype="f32", conv=False, bidir=False, chunks=0),   # no scratch
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c['dtype']}-{c['shape']}-bidir{int(c['bidir'])}-c{c['chunks']}")
def test_noalloc_matches_regular_entry_point(case):
    lib = _abi.load()
    B, D, L, N = case["shape"]
    dtype = case["dtype"]
    inp = synth.scan_inputs(B, D, L, N, dtype, conv_width=4 if case["conv"] else 0,
                            bidirectional=case["bidir"], seed=31)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    mk = lambda: (torch.empty(B, D, L, dtype=tdt, device="cuda"),
                  torch.empty(B, D, N, device="cuda"), torch.empty(B, D, N, device="cuda"))

    # regular entry point, caller-allocated workspace
    out_r, fs_r, fsr_r = mk()
    a, keep = _args(inp, dtype, conv=case["conv"], bidir=case["bidir"], chunks=case["chunks"],
                    out=out_r, fs=fs_r, fsr=fsr_r)
    n = ctypes.c_size_t()
    assert lib.ssm_selective_scan_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    assert n.value <= _abi.NOALLOC_SCRATCH_BYTES
    ws = torch.empty(max(n.value, 1), dtype=torch.uint8, device="cuda")
    a.workspace, a.workspace_bytes = ws.data_ptr(), n.value
    assert lib.ssm_selective_scan_fwd(ctypes.byref(a), _stream()) == 0

    # unrelated contents in the shared scratch: the same shape with other inputs
    other = synth.scan_inputs(B, D, L, N, dtype, conv_width=4 if case["conv"] else 0,
                              bidirectional=case["bidir"], seed=77)
    other["A"] = other["A"] * 0.37
    other["delta"] = other["delta"] + 1.5
    out_o, fs_o, fsr_o = mk()
    c, keep3 = _args(other, dtype, conv=case["conv"], bidir=case["bidir"], chunks=case["chunks"],
                     out=out_o, fs=fs_o, fsr=fsr_o)
    assert lib.ssm_selective_scan_fwd_noalloc(ctypes.byref(c), _stream()) == 0

    # the no-allocation entry point, twice in a row on fresh outputs
    for call in range(2):
        out_n, fs_n, fsr_n = mk()
        b, keep2 = _args(inp, dtype, conv=case["conv"], bidir=case["bidir"],
                         chunks=case["chunks"], out=out_n, fs=fs_n, fsr=fsr_n)
        status = lib.ssm_selective_scan_fwd_noalloc(ctypes.byref(b), _stream())
        assert status == 0, (lib.ssm_last_error_detail() or b"").decode()
        torch.cuda.synchronize()
        what = f"call {call + 1}"
        if dtype == "bf16":
            assert_bf16_ulp(host(out_n), host(out_r), what)
        else:
            assert_close(host(out_n), host(out_r), dtype, what)
        state_close(host(fs_n), host(fs_r), what + " final state")
        if case["bidir"]:
            state_close(host(fsr_n), host(fsr_r), what + " reverse final state")
    assert ssm.ssm_device_error() == 0


def test_noalloc_rejects_scratch_beyond_its_fixed_size():
    """A bf16 bidirectional call whose fp32 partial exceeds the fixed scratch is refused."""
    lib = _abi.load()
    B, D, L, N = 4, 64, 16384, 16           # partial: 4*64*16384*4 B = 16 MiB > 8 MiB
    inp = synth.scan_inputs(B, D, L, N, "bf16", bidirectional=True, seed=32)
    out = torch.full((B, D, L), 7.0, dtype=torch.bfloat16, device="cuda")
    fs = torch.zeros(B, D, N, device="cuda")
    fsr = torch.zeros(B, D, N, device="cuda")
    a, keep = _args(inp, "bf16", conv=False, bidir=True, chunks=0, out=out, fs=fs, fsr=fsr)
    status = lib.ssm_selective_scan_fwd_noalloc(ctypes.byref(a), _stream())
    assert status == _abi.STATUS_CODE["SSM_ERR_WORKSPACE"]
    assert b"scratch" in lib.ssm_last_error_detail()
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)             # nothing was launched
