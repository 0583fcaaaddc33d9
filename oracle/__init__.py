"""CPU oracle (double precision) for the selective-scan forward and the decode step.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the bench's CPU
baseline use it; the product path never imports it. The arithmetic lives in
``oracle.c`` (plain sequential C, built with gcc -O2, no fast-math); this module
only builds/loads that library and marshals numpy arrays.

``selective_scan_bidir`` composes the bidirectional variant (kanishk-sama.me
"ARM Selective-Scan Kernel", "What I built": forward scan plus the scan of the
flipped sequence) as the sum of a forward and a reverse call, each with its own
A, D and dt bias; u, delta, B, C and z are shared.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc -O2, IEEE double, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-std=c99",
                               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def load_library(path: str):
    """Open a compiled oracle library and declare its signatures."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    L = ctypes.c_long
    I = ctypes.c_int
    lib.oracle_causal_conv1d.argtypes = [P, P, P, P, L, L, L, I, I]
    lib.oracle_selective_scan.argtypes = [P, P, P, P, P, P, P, P, I, I, P, P, I, P, P, P, P,
                                          L, L, L, L, I]
    lib.oracle_state_update.argtypes = [P, P, P, P, P, P, P, P, P, P, I, P, P, I, P, L, L, L]
    for f in (lib.oracle_causal_conv1d, lib.oracle_selective_scan, lib.oracle_state_update):
        f.restype = None
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = load_library(build())
    return _lib


def _d(a):
    """Contiguous float64 copy (or None)."""
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def causal_conv1d(x, w, bias=None, apply_silu=True):
    """x (B, D, L), w (D, W), bias (D) -> (B, D, L)."""
    x, w, bias = _d(x), _d(w), _d(bias)
    Bsz, D, L = x.shape
    out = np.empty_like(x)
    _load().oracle_causal_conv1d(_p(x), _p(w), _p(bias), _p(out), Bsz, D, L, w.shape[1],
                                 int(bool(apply_silu)))
    return out


def head_A(A, dim, N):
    """A given per head, shape (nheads,): channel d belongs to head d // (dim // nheads)
    and all its N states decay with that head's scalar (paperlayer.ai summary of arXiv
    2603.09555, §3 Method, "State-space duality": A restricted to a scalar per head).
    Returns the equivalent (dim, N) matrix; a (dim, N) A is returned unchanged."""
    A = np.asarray(A, dtype=np.float64)
    if A.ndim == 2:
        return A
    nheads = A.shape[0]
    assert dim % nheads == 0, "dim must be a whole number of heads"
    return np.repeat(A, dim // nheads)[:, None] * np.ones((1, N))


def selective_scan(u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
                   reverse=False, conv_w=None, conv_b=None, h0=None, return_final_state=False,
                   conv_hist=None):
    """One-direction scan. u, delta, z (B, D, L); B, C (B, N, L), or time-invariant
    (D, N); A (D, N), or one scalar per head (nheads,).

    With ``conv_w`` (D, W) given, ``u`` is the pre-conv x and the scan input is
    silu(conv(x) + conv_b). ``h0`` (B, D, N) is the initial state; ``conv_hist``
    (B, D, W-1) holds the inputs before position 0, oldest first (forward only).
    Returns y (B, D, L) [and the final state (B, D, N)].
    """
    u, delta, B, C = _d(u), _d(delta), _d(B), _d(C)
    D, z, delta_bias, conv_w, conv_b, h0 = _d(D), _d(z), _d(delta_bias), _d(conv_w), _d(conv_b), _d(h0)
    conv_hist = _d(conv_hist)
    assert conv_hist is None or (conv_w is not None and not reverse)
    Bsz, Dm, L = u.shape
    shared = B.ndim == 2
    N = B.shape[1]
    A = _d(head_A(A, Dm, N))
    if shared:
        assert B.shape == (Dm, N) and C.shape == (Dm, N)
    else:
        assert B.shape == (Bsz, N, L) and C.shape == (Bsz, N, L)
    assert delta.shape == u.shape and A.shape == (Dm, N)
    out = np.empty_like(u)
    fs = np.empty((Bsz, Dm, N), dtype=np.float64)
    W = conv_w.shape[1] if conv_w is not None else 0
    _load().oracle_selective_scan(_p(u), _p(delta), _p(A), _p(B), _p(C), _p(D), _p(z),
                                  _p(delta_bias), int(bool(delta_softplus)), int(bool(reverse)),
                                  _p(conv_w), _p(conv_b), W, _p(h0), _p(conv_hist), _p(out),
                                  _p(fs), Bsz, Dm, L, N, int(shared))
    return (out, fs) if return_final_state else out


def conv_tail(x, W, conv_hist=None):
    """The last W inputs of the sequence conv_hist ++ x (zeros before either), oldest
    first: the conv state a decode step or a following scan continues from."""
    x = _d(x)
    Bsz, Dm, L = x.shape
    hist = np.zeros((Bsz, Dm, W - 1)) if conv_hist is None else _d(conv_hist)
    full = np.concatenate([np.zeros((Bsz, Dm, 1)), hist, x], axis=2)
    return full[:, :, -W:].copy()


def selective_scan_bidir(u, delta, A, B, C, D, z, delta_bias, A_rev, D_rev, delta_bias_rev,
                         delta_softplus=True, conv_w=None, conv_b=None, return_final_state=False):
    """Forward scan (A, D, delta_bias) plus reverse scan (A_rev, D_rev, delta_bias_rev)."""
    yf, hf = selective_scan(u, delta, A, B, C, D, z, delta_bias, delta_softplus, False,
                            conv_w, conv_b, return_final_state=True)
    yr, hr = selective_scan(u, delta, A_rev, B, C, D_rev, z, delta_bias_rev, delta_softplus, True,
                            conv_w, conv_b, return_final_state=True)
    y = yf + yr
    return (y, hf, hr) if return_final_state else y


def state_update(state, conv_state, x, dt, A, B, C, D=None, z=None, dt_bias=None,
                 dt_softplus=True, conv_w=None, conv_b=None):
    """One decode step. Returns (y (B, D), new_state, new_conv_state); inputs untouched.

    state (B, D, N); conv_state (B, D, W) newest last; x, dt, z (B, D); B, C (B, N);
    A (D, N), or one scalar per head (nheads,).
    """
    st = _d(state).copy()
    cs = _d(conv_state).copy() if conv_state is not None else None
    x, dt, B, C = _d(x), _d(dt), _d(B), _d(C)
    A = _d(head_A(A, st.shape[1], st.shape[2]))
    D, z, dt_bias, conv_w, conv_b = _d(D), _d(z), _d(dt_bias), _d(conv_w), _d(conv_b)
    Bsz, Dm, N = st.shape
    W = conv_w.shape[1] if conv_w is not None else 0
    out = np.empty((Bsz, Dm), dtype=np.float64)
    _load().oracle_state_update(_p(st), _p(cs), _p(x), _p(dt), _p(A), _p(B), _p(C), _p(D), _p(z),
                                _p(dt_bias), int(bool(dt_softplus)), _p(conv_w), _p(conv_b), W,
                                _p(out), Bsz, Dm, N)
    return out, st, cs


def scan_channels(inp: dict, chans, *, reverse=False, conv=False, final_state=False,
                  bidirectional=False, delta_softplus=True):
    """Oracle outputs for a sample of channels [(b, d), ...] of a full-size input dict.

    Each channel's scan is independent, so a sample is computed one channel row at
    a time from the same arrays the GPU received. Returns y (n, L) and, if asked,
    final states (n, N) [and reverse final states for bidirectional].
    """
    ys, hs, hrs = [], [], []
    Dm = inp["u"].shape[1]
    shared = inp["B"].ndim == 2
    N = inp["B"].shape[1]
    for b, d in chans:
        sl = lambda a: None if a is None else a[b:b + 1, d:d + 1]
        bc = (lambda k: inp[k][d:d + 1]) if shared else (lambda k: inp[k][b:b + 1])
        args = dict(u=sl(inp["u"]), delta=sl(inp["delta"]), B=bc("B"), C=bc("C"),
                    z=sl(inp.get("z")))

        def pd(k):
            if inp.get(k) is None:
                return None
            if k in ("A", "A_rev"):
                return head_A(inp[k], Dm, N)[d:d + 1]
            return inp[k][d:d + 1]
        cw = pd("conv_w") if conv else None
        cb = pd("conv_b") if conv else None
        if bidirectional:
            y, hf, hr = selective_scan_bidir(
                args["u"], args["delta"], pd("A"), args["B"], args["C"], pd("D"), args["z"],
                pd("delta_bias"), pd("A_rev"), pd("D_rev"), pd("delta_bias_rev"),
                delta_softplus, cw, cb, return_final_state=True)
            hrs.append(hr[0, 0])
        else:
            y, hf = selective_scan(args["u"], args["delta"], pd("A"), args["B"], args["C"],
                                   pd("D"), args["z"], pd("delta_bias"), delta_softplus, reverse,
                                   cw, cb, return_final_state=True)
        ys.append(y[0, 0])
        hs.append(hf[0, 0])
    res = [np.stack(ys)]
    if final_state:
        res.append(np.stack(hs))
        if bidirectional:
            res.append(np.stack(hrs))
    return res[0] if len(res) == 1 else tuple(res)
