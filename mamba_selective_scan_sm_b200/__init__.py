"""Mamba selective-scan forward and decode state update for B200 (sm_100a).

A thin binding over the C ABI in include/ssm.h: it takes torch CUDA tensors,
passes their device pointers and the current stream to libssm_b200.so, and
allocates the outputs (and the scan's workspace) through torch. Every step of
the computation runs in the library's kernels; there is no fallback, and a
missing library raises ``LibraryMissing``.

Functions carry the ABI's names:

* ``ssm_causal_conv1d_fwd(x, w, bias=None, apply_silu=True)``
* ``ssm_selective_scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, ...)``
* ``ssm_selective_state_update(state, conv_state, x, dt, A, B, C, ...)`` (in place)
"""
from __future__ import annotations

import ctypes

from . import _abi
from ._abi import LibraryMissing, SSMError, ScanArgs  # noqa: F401

__all__ = ["ssm_causal_conv1d_fwd", "ssm_selective_scan_fwd", "ssm_selective_scan_workspace_size",
           "ssm_selective_state_update", "ssm_device_error", "LibraryMissing", "SSMError", "ssm_wait_selftest"]


def _torch():
    import torch
    return torch


def _dtype_code(t):
    torch = _torch()
    if t.dtype == torch.float32:
        return _abi.SSM_F32
    if t.dtype == torch.bfloat16:
        return _abi.SSM_BF16
    raise TypeError(f"activations must be float32 or bfloat16, got {t.dtype}")


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr() if t.numel() else None


def _fp32(t, name):
    if t is not None and t.dtype != _torch().float32:
        raise TypeError(f"{name} must be float32")
    return _ptr(t)


def _stream(stream):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _position_stride(t, name):
    """Channel-last (batch, seqlen, width) view: its element stride between positions.
    The last axis must be dense and the batch rows seqlen positions apart."""
    if t is None:
        return 0
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    b, L, w = t.shape
    if t.numel() and (t.stride(2) != 1 or (b > 1 and t.stride(0) != L * t.stride(1))):
        raise ValueError(f"{name}: channel-last views need stride (seqlen*s, s, 1)")
    return t.stride(1)


def _dstate(A, B, channel_last):
    """d_state: from A (dim, dstate), or, with A given per head, from B."""
    if A.dim() == 2:
        return A.shape[1]
    if B.dim() == 2:                      # time-invariant (dim, dstate)
        return B.shape[1]
    return B.shape[2] if channel_last else B.shape[1]


def _view_ptr(t):
    return None if t is None or not t.numel() else t.data_ptr()


def _scan_args(u, delta, A, B, C, D, z, delta_bias, delta_softplus, reverse, conv_weight,
               conv_bias, A_rev, D_rev, delta_bias_rev, out, final_state, final_state_rev,
               num_chunks, channel_last=False):
    a = ScanArgs()
    a.dtype = _dtype_code(u)
    if channel_last:
        batch, seqlen, dim = u.shape
        a.channel_last = 1
        a.stride_u, a.stride_delta = _position_stride(u, "u"), _position_stride(delta, "delta")
        a.stride_z, a.stride_out = _position_stride(z, "z"), _position_stride(out, "out")
        if B.dim() == 3:
            a.stride_B, a.stride_C = _position_stride(B, "B"), _position_stride(C, "C")
        a.u, a.delta, a.z = (_view_ptr(t) for t in (u, delta, z))
    else:
        batch, dim, seqlen = u.shape
        a.u, a.delta, a.z = _ptr(u), _ptr(delta), _ptr(z)
    shared = B.dim() == 2                 # time-invariant B, C: fp32 (dim, dstate)
    if shared:
        a.B, a.C, a.bc_shared = _fp32(B, "B"), _fp32(C, "C"), 1
    else:
        a.B, a.C = (_view_ptr(B), _view_ptr(C)) if channel_last else (_ptr(B), _ptr(C))
    a.batch, a.dim, a.seqlen = batch, dim, seqlen
    a.dstate = _dstate(A, B, channel_last)
    a.a_heads = A.shape[0] if A.dim() == 1 else 0
    a.A, a.D, a.delta_bias = _fp32(A, "A"), _fp32(D, "D"), _fp32(delta_bias, "delta_bias")
    a.delta_softplus, a.reverse = int(bool(delta_softplus)), int(bool(reverse))
    a.conv_weight, a.conv_bias = _fp32(conv_weight, "conv_weight"), _fp32(conv_bias, "conv_bias")
    a.conv_width = conv_weight.shape[1] if conv_weight is not None else 0
    a.A_rev, a.D_rev = _fp32(A_rev, "A_rev"), _fp32(D_rev, "D_rev")
    a.delta_bias_rev = _fp32(delta_bias_rev, "delta_bias_rev")
    a.out = _view_ptr(out) if channel_last else _ptr(out)
    a.final_state, a.final_state_rev = _ptr(final_state), _ptr(final_state_rev)
    a.num_chunks = int(num_chunks)
    return a


def ssm_selective_scan_workspace_size(u, A, *, conv_weight=None, A_rev=None, num_chunks=0,
                                      reverse=False, seq_starts=None, channel_last=False,
                                      dstate=None, bc_shared=False):
    """Workspace bytes ssm_selective_scan_fwd needs for these shapes (host-only query).
    With A given per head (a 1-D tensor), ``dstate`` must be given."""
    lib = _abi.load()
    a = ScanArgs()
    a.dtype = _dtype_code(u)
    if channel_last:
        a.batch, a.seqlen, a.dim = u.shape
        a.channel_last = 1
    else:
        a.batch, a.dim, a.seqlen = u.shape
    if A.dim() == 1:
        if dstate is None:
            raise ValueError("A given per head: pass dstate")
        a.dstate, a.a_heads = int(dstate), A.shape[0]
    else:
        a.dstate = A.shape[1]
    a.bc_shared = int(bool(bc_shared))
    a.reverse = int(bool(reverse))
    a.A_rev = 1 if A_rev is not None else None
    a.conv_weight = 1 if conv_weight is not None else None
    a.conv_width = conv_weight.shape[1] if conv_weight is not None else 0
    a.num_chunks = int(num_chunks)
    if seq_starts is not None:
        a.seq_starts, a.num_seqs = 1, seq_starts.numel() - 1     # only its presence is read
    n = ctypes.c_size_t()
    _abi.check(lib, lib.ssm_selective_scan_workspace_size(ctypes.byref(a), ctypes.byref(n)))
    return n.value


def ssm_selective_scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                           delta_softplus=True, reverse=False, conv_weight=None, conv_bias=None,
                           A_rev=None, D_rev=None, delta_bias_rev=None, *, out=None,
                           return_final_state=False, final_state=None, final_state_rev=None,
                           num_chunks=0, workspace=None, stream=None, initial_state=None,
                           conv_history=None, conv_state_out=None, return_conv_state=False,
                           seq_starts=None, channel_last=False):
    """Selective-scan forward (see include/ssm.h). Layouts: u, delta, z (batch, dim, seqlen);
    B, C (batch, dstate, seqlen), or fp32 (dim, dstate) for time-invariant B/C; A (dim,
    dstate) fp32, or (nheads,) for one scalar per head (d_state then comes from B). With
    ``conv_weight`` (dim, width), ``u`` is the pre-conv x. With ``A_rev`` (shaped as A) the
    result is the bidirectional sum.

    ``final_state`` / ``final_state_rev`` may be given as preallocated fp32 outputs
    (batch, dim, dstate); they are written whenever given. A forward scan continues a
    sequence from ``initial_state`` (batch, dim, dstate) fp32 and ``conv_history``
    (batch, dim, width - 1); ``conv_state_out`` (batch, dim, width), allocated when
    ``return_conv_state``, receives the conv state the next call continues from.
    ``seq_starts`` (int32, num_seqs + 1 offsets; batch 1) packs several sequences along the
    sequence axis: final_state is then (num_seqs, dim, dstate) and the conv state
    (num_seqs, dim, width). ``channel_last``: u, delta, z, out are (batch, seqlen, dim)
    and B, C (batch, seqlen, dstate), each possibly a view with a position stride
    (e.g. x and z halves of one in_proj output); ``out`` defaults to a dense tensor.
    Returns ``out``, or a tuple ``(out[, final_state[, final_state_rev]][, conv_state])``.
    """
    torch = _torch()
    lib = _abi.load()
    if out is None:
        out = (torch.empty(u.shape, dtype=u.dtype, device=u.device) if channel_last
               else torch.empty_like(u))
    fs, fsr = final_state, final_state_rev
    nseq = 0 if seq_starts is None else seq_starts.numel() - 1
    if seq_starts is not None and seq_starts.dtype != torch.int32:
        raise TypeError("seq_starts must be int32")
    rows = nseq if seq_starts is not None else u.shape[0]
    dim = u.shape[2] if channel_last else u.shape[1]
    if return_final_state:
        shp = (rows, dim, _dstate(A, B, channel_last))
        if fs is None:
            fs = torch.empty(shp, dtype=torch.float32, device=u.device)
        if A_rev is not None and fsr is None:
            fsr = torch.empty(shp, dtype=torch.float32, device=u.device)
    cs = conv_state_out
    if return_conv_state and cs is None:
        cs = torch.empty(rows, dim, conv_weight.shape[1], dtype=u.dtype, device=u.device)
    a = _scan_args(u, delta, A, B, C, D, z, delta_bias, delta_softplus, reverse, conv_weight,
                   conv_bias, A_rev, D_rev, delta_bias_rev, out, fs, fsr, num_chunks,
                   channel_last)
    a.initial_state = _fp32(initial_state, "initial_state")
    a.conv_history = _ptr(conv_history)
    a.conv_state_out = _ptr(cs)
    a.seq_starts, a.num_seqs = _ptr(seq_starts), nseq
    n = ctypes.c_size_t()
    _abi.check(lib, lib.ssm_selective_scan_workspace_size(ctypes.byref(a), ctypes.byref(n)))
    if n.value:
        if workspace is None or workspace.numel() < n.value:
            workspace = torch.empty(n.value, dtype=torch.uint8, device=u.device)
        a.workspace, a.workspace_bytes = _ptr(workspace), n.value
    _abi.check(lib, lib.ssm_selective_scan_fwd(ctypes.byref(a), _stream(stream)))
    res = [out]
    if return_final_state:
        res += [fs, fsr] if A_rev is not None else [fs]
    if return_conv_state:
        res.append(cs)
    return res[0] if len(res) == 1 else tuple(res)


def ssm_causal_conv1d_fwd(x, w, bias=None, apply_silu=True, *, out=None, stream=None):
    """Causal depthwise conv1d (+ SiLU). x (batch, dim, seqlen); w (dim, width) fp32."""
    torch = _torch()
    lib = _abi.load()
    if out is None:
        out = torch.empty_like(x)
    batch, dim, seqlen = x.shape
    _abi.check(lib, lib.ssm_causal_conv1d_fwd(_ptr(x), _fp32(w, "w"), _fp32(bias, "bias"),
                                              _ptr(out), batch, dim, seqlen, w.shape[1],
                                              int(bool(apply_silu)), _dtype_code(x),
                                              _stream(stream)))
    return out


def ssm_selective_state_update(state, conv_state, x, dt, A, B, C, D=None, z=None, dt_bias=None,
                               dt_softplus=True, conv_weight=None, conv_bias=None, *, out=None,
                               stream=None):
    """One decode step, in place on ``state`` (batch, dim, dstate) fp32 and ``conv_state``
    (batch, dim, width). x, dt, z (batch, dim); B, C (batch, dstate); A (dim, dstate), or
    (nheads,) for one scalar per head; dstate up to 128. Returns y (batch, dim)."""
    torch = _torch()
    lib = _abi.load()
    if out is None:
        out = torch.empty_like(x)
    batch, dim, dstate = state.shape
    width = conv_weight.shape[1] if conv_weight is not None else 0
    if A.dim() == 1 or dstate > 16:
        # A per head (a 1-D tensor, one scalar per head) or d_state above 16
        a = _abi.UpdateArgs()
        a.dtype, a.batch, a.dim, a.dstate = _dtype_code(x), batch, dim, dstate
        a.state, a.conv_state, a.x, a.dt = _fp32(state, "state"), _ptr(conv_state), _ptr(x), _ptr(dt)
        a.A, a.B_t, a.C_t, a.D = _fp32(A, "A"), _ptr(B), _ptr(C), _fp32(D, "D")
        a.z, a.dt_bias, a.dt_softplus = _ptr(z), _fp32(dt_bias, "dt_bias"), int(bool(dt_softplus))
        a.conv_weight, a.conv_bias = _fp32(conv_weight, "conv_weight"), _fp32(conv_bias, "conv_bias")
        a.conv_width, a.out = width, _ptr(out)
        a.a_heads = A.shape[0] if A.dim() == 1 else 0
        _abi.check(lib, lib.ssm_selective_state_update_ex(ctypes.byref(a), _stream(stream)))
        return out
    _abi.check(lib, lib.ssm_selective_state_update(
        _fp32(state, "state"), _ptr(conv_state), _ptr(x), _ptr(dt), _fp32(A, "A"), _ptr(B),
        _ptr(C), _fp32(D, "D"), _ptr(z), _fp32(dt_bias, "dt_bias"), int(bool(dt_softplus)),
        _fp32(conv_weight, "conv_weight"), _fp32(conv_bias, "conv_bias"), width, _ptr(out),
        batch, dim, dstate, _dtype_code(x), _stream(stream)))
    return out


def ssm_device_error(stream=None) -> int:
    """Read and clear the library's device error word (synchronises the stream)."""
    lib = _abi.load()
    code = ctypes.c_int32()
    _abi.check(lib, lib.ssm_device_error(ctypes.byref(code), _stream(stream)))
    return code.value


def ssm_wait_selftest(limit_ns=1_000_000, stream=None) -> None:
    """Enqueue the failure-path self-test: one bounded wait that runs out after
    ``limit_ns`` and sets the device error word (read it with ssm_device_error)."""
    lib = _abi.load()
    _abi.check(lib, lib.ssm_wait_selftest(int(limit_ns), _stream(stream)))
