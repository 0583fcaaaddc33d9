"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each check compares the oracle with a closed form, a hand-worked fixture, a
library routine, a 50-digit brute-force evaluation or an invariant, chosen so
that a plausible slip in the oracle (a dropped term, a flipped sign or tap, a
transposed B/C, an off-by-one in the recurrence, the skip term outside the gate)
fails at least one of them.
"""
import json
import math
import os

import mpmath
import numpy as np
import pytest
import scipy.special
import torch

import oracle
from mamba_selective_scan_sm_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _arr(x):
    return None if x is None else np.asarray(x, dtype=np.float64)


def _silu(v):
    return v * scipy.special.expit(v)


def _softplus(v):
    return np.logaddexp(0.0, v)


def _rand_case(rng, B=2, D=3, L=7, N=4, conv=0):
    c = dict(u=rng.standard_normal((B, D, L)), delta=0.5 * rng.standard_normal((B, D, L)),
             z=rng.standard_normal((B, D, L)), B=rng.standard_normal((B, N, L)),
             C=rng.standard_normal((B, N, L)), A=-rng.uniform(0.2, 3.0, (D, N)),
             D=rng.standard_normal(D), delta_bias=rng.uniform(-3, 0.5, D))
    if conv:
        c["conv_w"] = 0.5 * rng.standard_normal((D, conv))
        c["conv_b"] = 0.3 * rng.standard_normal(D)
    return c


# ---------------------------------------------------------------- fixtures ---

@pytest.mark.parametrize("name", ["l1_readout.json", "running_sum.json", "geometric_decay.json"])
def test_golden_scan(name):
    g = _golden(name)
    tol = g.get("tolerance", 1e-15)
    y, h = oracle.selective_scan(_arr(g["u"]), _arr(g["delta"]), _arr(g["A"]), _arr(g["B"]),
                                 _arr(g["C"]), _arr(g["D"]), _arr(g["z"]), _arr(g["delta_bias"]),
                                 g["delta_softplus"], False, return_final_state=True)
    np.testing.assert_allclose(y, _arr(g["y"]), rtol=tol, atol=tol)
    np.testing.assert_allclose(h, _arr(g["final_state"]), rtol=tol, atol=tol)
    if "y_reverse" in g:
        y, h = oracle.selective_scan(_arr(g["u"]), _arr(g["delta"]), _arr(g["A"]), _arr(g["B"]),
                                     _arr(g["C"]), _arr(g["D"]), _arr(g["z"]),
                                     _arr(g["delta_bias"]), g["delta_softplus"], True,
                                     return_final_state=True)
        np.testing.assert_allclose(y, _arr(g["y_reverse"]), rtol=tol, atol=tol)
        np.testing.assert_allclose(h, _arr(g["final_state_reverse"]), rtol=tol, atol=tol)


def test_golden_bidirectional():
    """Forward and reverse directions with their own A, D and dt bias, summed
    (hand-derived fixture in which exchanging any of them changes the sum)."""
    g = _golden("bidirectional_sum.json")
    tol = g["tolerance"]
    y, hf, hr = oracle.selective_scan_bidir(
        _arr(g["u"]), _arr(g["delta"]), _arr(g["A"]), _arr(g["B"]), _arr(g["C"]), _arr(g["D"]),
        _arr(g["z"]), _arr(g["delta_bias"]), _arr(g["A_rev"]), _arr(g["D_rev"]),
        _arr(g["delta_bias_rev"]), g["delta_softplus"], return_final_state=True)
    np.testing.assert_allclose(y, _arr(g["y"]), rtol=tol, atol=tol)
    np.testing.assert_allclose(hf, _arr(g["final_state"]), rtol=tol, atol=tol)
    np.testing.assert_allclose(hr, _arr(g["final_state_rev"]), rtol=tol, atol=tol)


def test_golden_conv():
    g = _golden("conv_orientation.json")
    out = oracle.causal_conv1d(_arr(g["x"]), _arr(g["w"]), _arr(g["bias"]), g["apply_silu"])
    np.testing.assert_array_equal(out, _arr(g["out"]))


def test_golden_decode():
    g = _golden("decode_step.json")
    y, st, _ = oracle.state_update(_arr(g["state"]), None, _arr(g["x"]), _arr(g["dt"]),
                                   _arr(g["A"]), _arr(g["B"]), _arr(g["C"]), _arr(g["D"]),
                                   _arr(g["z"]), _arr(g["dt_bias"]), g["dt_softplus"])
    np.testing.assert_array_equal(y, _arr(g["y"]))
    np.testing.assert_array_equal(st, _arr(g["state_after"]))
    # conv-state shift: newest input appended on the right
    w = np.array([[0.25, 0.75]])
    _, _, cs = oracle.state_update(_arr(g["state"]), _arr(g["conv_state"]), _arr(g["conv_x"]),
                                   _arr(g["dt"]), _arr(g["A"]), _arr(g["B"]), _arr(g["C"]),
                                   conv_w=w, conv_b=np.zeros(1), dt_softplus=False)
    np.testing.assert_array_equal(cs, _arr(g["conv_state_after"]))


# ------------------------------------------------------------ closed forms ---

@pytest.mark.parametrize("softplus", [False, True])
@pytest.mark.parametrize("gate", [False, True])
def test_A_zero_is_running_sum(softplus, gate):
    """A = 0: h_t = sum_{s<=t} delta_s B_s u_s (numpy cumsum), then y = C.h + D u, times silu(z)."""
    rng = np.random.default_rng(1)
    c = _rand_case(rng, B=2, D=3, L=37, N=5)
    A0 = np.zeros_like(c["A"])
    z = c["z"] if gate else None
    y, h = oracle.selective_scan(c["u"], c["delta"], A0, c["B"], c["C"], c["D"], z,
                                 c["delta_bias"], softplus, False, return_final_state=True)
    dl = c["delta"] + c["delta_bias"][None, :, None]
    if softplus:
        dl = _softplus(dl)
    dbu = dl[:, :, None, :] * c["B"][:, None, :, :] * c["u"][:, :, None, :]   # (B, D, N, L)
    hs = np.cumsum(dbu, axis=-1)
    yr = np.einsum("bnl,bdnl->bdl", c["C"], hs) + c["D"][None, :, None] * c["u"]
    if gate:
        yr = yr * _silu(c["z"])
    np.testing.assert_allclose(y, yr, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(h, hs[..., -1], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("reverse", [False, True])
def test_constant_inputs_geometric_series(reverse):
    """Constant delta, B, C, u: h_t = delta B u (1 - a^(k+1)) / (1 - a), a = exp(delta A),
    k = number of steps taken before t."""
    L, N = 50, 3
    dl, Bv, Cv, uv, Dv = 0.37, np.array([0.7, -1.2, 2.0]), np.array([1.5, 0.4, -0.9]), 1.3, 0.6
    A = np.array([[-0.5, -1.7, -3.1]])
    u = np.full((1, 1, L), uv)
    delta = np.full((1, 1, L), dl)
    Bm = np.repeat(Bv[None, :, None], L, axis=2)
    Cm = np.repeat(Cv[None, :, None], L, axis=2)
    y, h = oracle.selective_scan(u, delta, A, Bm, Cm, np.array([Dv]), None, None, False, reverse,
                                 return_final_state=True)
    a = np.exp(dl * A[0])
    k = np.arange(L)[::-1] if reverse else np.arange(L)
    hs = dl * Bv[:, None] * uv * (1 - a[:, None] ** (k[None, :] + 1)) / (1 - a[:, None])
    yr = (Cv[:, None] * hs).sum(0) + Dv * uv
    np.testing.assert_allclose(y[0, 0], yr, rtol=1e-13)
    np.testing.assert_allclose(h[0, 0], dl * Bv * uv * (1 - a ** L) / (1 - a), rtol=1e-13)


def test_seqlen_one_readout():
    """L = 1: y = (sum_n C_n delta B_n u + D u) silu(z), delta = softplus(dt + bias)."""
    rng = np.random.default_rng(2)
    c = _rand_case(rng, B=3, D=4, L=1, N=6)
    y, h = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                                 c["delta_bias"], True, False, return_final_state=True)
    dl = _softplus(c["delta"][..., 0] + c["delta_bias"][None])
    hr = dl[:, :, None] * c["B"][:, None, :, 0] * c["u"][..., 0][:, :, None]
    yr = (np.einsum("bn,bdn->bd", c["C"][..., 0], hr) + c["D"][None] * c["u"][..., 0]) \
        * _silu(c["z"][..., 0])
    np.testing.assert_allclose(y[..., 0], yr, rtol=1e-13)
    np.testing.assert_allclose(h, hr, rtol=1e-13)


def test_softplus_zero_is_ln2_and_silu_zero_is_zero():
    """delta = softplus(0) = ln 2 (A = 0, B = C = u = 1, N = 1: y = delta); silu(0) = 0 kills y."""
    one = np.ones((1, 1, 1))
    y = oracle.selective_scan(one, np.zeros((1, 1, 1)), np.zeros((1, 1)), one, one, None, None,
                              np.zeros(1), True)
    assert abs(y[0, 0, 0] - math.log(2.0)) < 1e-15
    y = oracle.selective_scan(one, np.zeros((1, 1, 1)), np.zeros((1, 1)), one, one, None,
                              np.zeros((1, 1, 1)), np.zeros(1), True)
    assert y[0, 0, 0] == 0.0


# -------------------------------------------------------- brute force, L<=8 ---

def _mp_silu(v):
    return v / (1 + mpmath.exp(-v))


@pytest.mark.parametrize("conv", [0, 4])
@pytest.mark.parametrize("reverse", [False, True])
def test_bruteforce_50_digits(conv, reverse):
    """h_t = sum_{s<=t} (prod_{r=s+1..t} dA_r) dBu_s as explicit products at 50 digits."""
    mpmath.mp.dps = 50
    rng = np.random.default_rng(3 + conv + int(reverse))
    Bsz, D, L, N = 1, 2, 8, 3
    c = _rand_case(rng, Bsz, D, L, N, conv=conv)
    y = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                              c["delta_bias"], True, reverse, c.get("conv_w"), c.get("conv_b"))
    for d in range(D):
        x = [mpmath.mpf(float(v)) for v in c["u"][0, d]]
        order = list(range(L))[::-1] if reverse else list(range(L))
        xs = [x[t] for t in order]                     # sequence as the scan walks it
        if conv:
            w = [mpmath.mpf(float(v)) for v in c["conv_w"][d]]
            us = []
            for i in range(L):
                acc = mpmath.mpf(float(c["conv_b"][d]))
                for k in range(conv):
                    s = i - (conv - 1) + k
                    if s >= 0:
                        acc += w[k] * xs[s]
                us.append(_mp_silu(acc))
        else:
            us = xs
        dts = [mpmath.log(1 + mpmath.exp(mpmath.mpf(float(c["delta"][0, d, t]))
                                         + mpmath.mpf(float(c["delta_bias"][d])))) for t in order]
        for i, t in enumerate(order):
            yt = mpmath.mpf(0)
            for n in range(N):
                An = mpmath.mpf(float(c["A"][d, n]))
                hn = mpmath.mpf(0)
                for s in range(i + 1):
                    prod = mpmath.mpf(1)
                    for r in range(s + 1, i + 1):
                        prod *= mpmath.exp(dts[r] * An)
                    hn += prod * dts[s] * mpmath.mpf(float(c["B"][0, n, order[s]])) * us[s]
                yt += mpmath.mpf(float(c["C"][0, n, t])) * hn
            yt += mpmath.mpf(float(c["D"][d])) * us[i]
            yt *= _mp_silu(mpmath.mpf(float(c["z"][0, d, t])))
            assert abs(float(yt) - y[0, d, t]) <= 1e-13 * max(1.0, abs(float(yt))), (d, t)


# ------------------------------------------------------ library routines ---

@pytest.mark.parametrize("W", [2, 3, 4])
def test_conv_matches_torch_conv1d(W):
    """Depthwise Conv1d with padding W-1, first L outputs kept (the causal reading)."""
    rng = np.random.default_rng(4)
    Bsz, D, L = 2, 5, 19
    x, w, b = rng.standard_normal((Bsz, D, L)), rng.standard_normal((D, W)), rng.standard_normal(D)
    ref = torch.nn.functional.conv1d(torch.from_numpy(x), torch.from_numpy(w)[:, None, :],
                                     torch.from_numpy(b), padding=W - 1, groups=D)[..., :L].numpy()
    np.testing.assert_allclose(oracle.causal_conv1d(x, w, b, False), ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.causal_conv1d(x, w, b, True), _silu(ref), rtol=1e-12,
                               atol=1e-12)


def test_fused_conv_scan_equals_conv_then_scan():
    rng = np.random.default_rng(5)
    c = _rand_case(rng, 2, 3, 23, 4, conv=4)
    y1 = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                               c["delta_bias"], True, False, c["conv_w"], c["conv_b"])
    u = oracle.causal_conv1d(c["u"], c["conv_w"], c["conv_b"], True)
    y2 = oracle.selective_scan(u, c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                               c["delta_bias"], True, False)
    np.testing.assert_allclose(y1, y2, rtol=1e-14, atol=1e-14)


# ------------------------------------------------------------- invariants ---

@pytest.mark.parametrize("conv", [0, 4])
def test_reverse_is_flip_forward_flip(conv):
    rng = np.random.default_rng(6)
    c = _rand_case(rng, 2, 3, 29, 4, conv=conv)
    yr, hr = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                                   c["delta_bias"], True, True, c.get("conv_w"), c.get("conv_b"),
                                   return_final_state=True)
    f = lambda a: None if a is None else a[..., ::-1]
    yf, hf = oracle.selective_scan(f(c["u"]), f(c["delta"]), c["A"], f(c["B"]), f(c["C"]), c["D"],
                                   f(c["z"]), c["delta_bias"], True, False, c.get("conv_w"),
                                   c.get("conv_b"), return_final_state=True)
    np.testing.assert_allclose(yr, yf[..., ::-1], rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(hr, hf, rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("N,heads", [(4, 0), (64, 3)])
def test_decode_repeated_equals_scan(N, heads):
    """L decode steps from zero state and zero conv history reproduce the fused-conv scan
    (with A per head and d_state 64 too: the scan's per-head form is pinned by the dual
    form above)."""
    rng = np.random.default_rng(7)
    Bsz, D, L, W = 2, 3, 17, 4
    c = _rand_case(rng, Bsz, D, L, N, conv=W)
    if heads:
        c["A"] = -rng.uniform(0.2, 2.0, heads)         # one head per channel here
    y, h = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                                 c["delta_bias"], True, False, c["conv_w"], c["conv_b"],
                                 return_final_state=True)
    st = np.zeros((Bsz, D, N))
    cs = np.zeros((Bsz, D, W))
    for t in range(L):
        yt, st, cs = oracle.state_update(st, cs, c["u"][..., t], c["delta"][..., t], c["A"],
                                         c["B"][..., t], c["C"][..., t], c["D"], c["z"][..., t],
                                         c["delta_bias"], True, c["conv_w"], c["conv_b"])
        np.testing.assert_allclose(yt, y[..., t], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(st, h, rtol=1e-12, atol=1e-13)


def test_linear_in_u_without_conv_and_gate():
    rng = np.random.default_rng(8)
    c = _rand_case(rng, 1, 3, 31, 4)
    u2 = rng.standard_normal(c["u"].shape)
    run = lambda u: oracle.selective_scan(u, c["delta"], c["A"], c["B"], c["C"], c["D"], None,
                                          c["delta_bias"], True)
    np.testing.assert_allclose(run(2.5 * c["u"] - 0.75 * u2), 2.5 * run(c["u"]) - 0.75 * run(u2),
                               rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("reverse", [False, True])
def test_causality(reverse):
    rng = np.random.default_rng(9)
    c = _rand_case(rng, 1, 2, 40, 4, conv=4)
    t0 = 17
    run = lambda cc: oracle.selective_scan(cc["u"], cc["delta"], cc["A"], cc["B"], cc["C"], cc["D"],
                                           cc["z"], cc["delta_bias"], True, reverse,
                                           cc["conv_w"], cc["conv_b"])
    y0 = run(c)
    for key in ("u", "delta", "B", "C", "z"):
        c2 = dict(c)
        c2[key] = c[key].copy()
        c2[key][..., t0] += 1.0
        y1 = run(c2)
        same = slice(t0 + 1, None) if reverse else slice(0, t0)
        np.testing.assert_array_equal(y1[..., same], y0[..., same])
        assert np.all(y1[..., t0] != y0[..., t0]) or key == "z", key


def test_zero_B_or_C_leaves_skip_times_gate():
    rng = np.random.default_rng(10)
    c = _rand_case(rng, 2, 3, 13, 4)
    ref = c["D"][None, :, None] * c["u"] * _silu(c["z"])
    for kill in ("B", "C"):
        cc = dict(c)
        cc[kill] = np.zeros_like(c[kill])
        y = oracle.selective_scan(cc["u"], cc["delta"], cc["A"], cc["B"], cc["C"], cc["D"], cc["z"],
                                  cc["delta_bias"], True)
        np.testing.assert_allclose(y, ref, rtol=1e-14, atol=1e-15)


def test_conv_one_hot_taps():
    rng = np.random.default_rng(11)
    x = rng.standard_normal((1, 2, 12))
    w = np.zeros((2, 4))
    w[:, 3] = 1.0                                   # newest tap: identity
    np.testing.assert_array_equal(oracle.causal_conv1d(x, w, None, False), x)
    w = np.zeros((2, 4))
    w[:, 0] = 1.0                                   # oldest tap: shift by W-1, zero fill
    out = oracle.causal_conv1d(x, w, None, False)
    np.testing.assert_array_equal(out[..., 3:], x[..., :-3])
    np.testing.assert_array_equal(out[..., :3], 0.0)


def test_bidirectional_palindrome():
    """Same parameters both ways and a palindromic sequence give a palindromic output."""
    rng = np.random.default_rng(12)
    c = _rand_case(rng, 1, 3, 21, 4, conv=4)
    pal = lambda a: np.concatenate([a[..., :11], a[..., :10][..., ::-1]], axis=-1)
    for k in ("u", "delta", "B", "C", "z"):
        c[k] = pal(c[k])
    y = oracle.selective_scan_bidir(c["u"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                                    c["delta_bias"], c["A"], c["D"], c["delta_bias"], True,
                                    c["conv_w"], c["conv_b"])
    np.testing.assert_allclose(y, y[..., ::-1], rtol=1e-13, atol=1e-13)


def test_two_pass_chunk_carry_matches_sequential():
    """Chunk summaries (P_c = exp(A sum delta), S_c = state from zero), the carry
    H_c = P_c H_{c-1} + S_c, and a rescan of each chunk from H_{c-1} give the
    sequential result: the algebra the chunk-parallel GPU path relies on."""
    rng = np.random.default_rng(13)
    c = _rand_case(rng, 2, 3, 60, 4)
    y, h = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                                 c["delta_bias"], True, False, return_final_state=True)
    bounds = [0, 13, 31, 32, 60]
    H = np.zeros((2, 3, 4))
    ys = []
    for c0, c1 in zip(bounds[:-1], bounds[1:]):
        sl = lambda a: a[..., c0:c1]
        yc = oracle.selective_scan(sl(c["u"]), sl(c["delta"]), c["A"], sl(c["B"]), sl(c["C"]),
                                   c["D"], sl(c["z"]), c["delta_bias"], True, False, h0=H)
        _, S = oracle.selective_scan(sl(c["u"]), sl(c["delta"]), c["A"], sl(c["B"]), sl(c["C"]),
                                     c["D"], sl(c["z"]), c["delta_bias"], True, False,
                                     return_final_state=True)
        dsum = _softplus(sl(c["delta"]) + c["delta_bias"][None, :, None]).sum(-1)
        P = np.exp(dsum[..., None] * c["A"][None])
        H = P * H + S
        ys.append(yc)
    np.testing.assert_allclose(np.concatenate(ys, axis=-1), y, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(H, h, rtol=1e-11, atol=1e-12)


# ------------------------------------------------ continuing a sequence ---

def _scan(c, sl=lambda a: a, **kw):
    return oracle.selective_scan(sl(c["u"]), sl(c["delta"]), c["A"], sl(c["B"]), sl(c["C"]),
                                 c["D"], sl(c["z"]), c["delta_bias"], True, False,
                                 c.get("conv_w"), c.get("conv_b"), return_final_state=True, **kw)


@pytest.mark.parametrize("W", [2, 3, 4])
def test_conv_history_is_the_conv_of_the_joined_sequence(W):
    """The scan input with a conv history equals the plain causal conv (pinned against
    torch above) of history ++ x: run the scan over the joined sequence with B = 0 on the
    history positions (they then leave the zero state untouched) and drop their outputs."""
    rng = np.random.default_rng(15)
    c = _rand_case(rng, 2, 3, 19, 4, conv=W)
    hist = rng.standard_normal((2, 3, W - 1))
    y, h = _scan(c, conv_hist=hist)
    j = dict(c)
    pad = lambda a, v: np.concatenate([v, a], axis=-1)
    j["u"] = pad(c["u"], hist)
    for k in ("delta", "z", "C"):
        j[k] = pad(c[k], rng.standard_normal(c[k].shape[:-1] + (W - 1,)))
    j["B"] = pad(c["B"], np.zeros((2, 4, W - 1)))
    yj, hj = _scan(j)
    np.testing.assert_array_equal(y, yj[..., W - 1:])
    np.testing.assert_array_equal(h, hj)
    # torch's conv1d over the joined sequence gives the same scan input
    xj = torch.from_numpy(j["u"])
    ref = torch.nn.functional.conv1d(xj, torch.from_numpy(c["conv_w"])[:, None, :],
                                     torch.from_numpy(c["conv_b"]), padding=W - 1,
                                     groups=3)[..., W - 1:W - 1 + 19].numpy()
    y_unfused, _ = oracle.selective_scan(_silu(ref), c["delta"], c["A"], c["B"], c["C"], c["D"],
                                         c["z"], c["delta_bias"], True, False,
                                         return_final_state=True)
    np.testing.assert_allclose(y, y_unfused, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("cuts", [(1,), (2,), (3,), (5,), (20,), (36,), (2, 3), (1, 2, 30)])
def test_split_sequence_continues_from_state_and_history(cuts):
    """Scanning a sequence in pieces, each from the previous piece's final state and the
    last W-1 inputs before it, reproduces the one-piece scan (pieces shorter than W-1
    included, so the history spans pieces)."""
    rng = np.random.default_rng(16)
    W, L = 4, 37
    c = _rand_case(rng, 2, 3, L, 5, conv=W)
    y, h = _scan(c)
    bounds = [0, *cuts, L]
    ys, st, hist = [], None, None
    for a, b in zip(bounds[:-1], bounds[1:]):
        sl = lambda v: v[..., a:b]
        yp, st = _scan(c, sl, h0=st, conv_hist=hist)
        hist = oracle.conv_tail(sl(c["u"]), W, hist)[..., 1:]
        ys.append(yp)
    np.testing.assert_allclose(np.concatenate(ys, axis=-1), y, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(st, h, rtol=1e-12, atol=1e-12)


def test_decode_continues_a_scan():
    """Decode steps from a scan's final state and conv tail reproduce the rest of the
    one-piece scan."""
    rng = np.random.default_rng(17)
    W, L, k = 4, 25, 9
    c = _rand_case(rng, 2, 3, L, 4, conv=W)
    y, h = _scan(c)
    _, st = _scan(c, lambda v: v[..., :k])
    cs = oracle.conv_tail(c["u"][..., :k], W)
    for t in range(k, L):
        yt, st, cs = oracle.state_update(st, cs, c["u"][..., t], c["delta"][..., t], c["A"],
                                         c["B"][..., t], c["C"][..., t], c["D"], c["z"][..., t],
                                         c["delta_bias"], True, c["conv_w"], c["conv_b"])
        np.testing.assert_allclose(yt, y[..., t], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(st, h, rtol=1e-12, atol=1e-13)


def test_conv_tail_layout():
    """conv_tail: the last W inputs of history ++ x, zeros before both, oldest first."""
    x = np.arange(1, 6, dtype=np.float64).reshape(1, 1, 5)           # 1..5
    np.testing.assert_array_equal(oracle.conv_tail(x, 4), [[[2, 3, 4, 5]]])
    np.testing.assert_array_equal(oracle.conv_tail(x[..., :2], 4), [[[0, 0, 1, 2]]])
    np.testing.assert_array_equal(oracle.conv_tail(x[..., :1], 4, np.array([[[7, 8, 9]]])),
                                  [[[7, 8, 9, 1]]])


def test_oracle_consumes_bf16_rounded_inputs():
    """The synthetic generator rounds to bf16 first; the rounding is nearest-even."""
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, -2.0 ** -130, 3.0e38], dtype=np.float32)
    r = synth.round_bf16(x)
    t = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(r, t)
    big = np.random.default_rng(14).standard_normal(100000).astype(np.float32)
    np.testing.assert_array_equal(synth.round_bf16(big),
                                  torch.from_numpy(big).to(torch.bfloat16).float().numpy())


# ------------------------------------------- heads, time-invariant B/C, large N ---
# State-space duality (paperlayer.ai summary of arXiv 2603.09555, §3 Method, "State-space
# duality" and "Chunked recurrence"): with A diagonal the recurrence unrolls to
#   h_t[n] = sum_{s<=t} exp(sum_{r=s+1..t} delta_r A[n]) delta_s u_s B_s[n],
# so y = sum_n (M_n o C[:, n] B[:, n]^T) (delta u) with the lower-triangular decay
# matrix M_n[t, s] = exp(cum_n[t] - cum_n[s]). The pins below evaluate that quadratic
# form with numpy matrix products: no recurrence, no loop over time.

def _dual_form(u, dl, A_dn, Bt, Ct, Dv, z):
    """One channel. u, dl, z (L,); A_dn (N,); Bt, Ct (L, N). Returns y (L,), h_L (N,)."""
    L, N = Bt.shape
    x = dl * u
    tri = np.tril(np.ones((L, L), dtype=bool))
    y = np.zeros(L)
    hL = np.zeros(N)
    for n in range(N):
        cum = np.cumsum(dl * A_dn[n])
        M = np.where(tri, np.exp(np.where(tri, cum[:, None] - cum[None, :], 0.0)), 0.0)
        y += (M * np.outer(Ct[:, n], Bt[:, n])) @ x
        hL[n] = (M[-1] * Bt[:, n]) @ x
    if Dv is not None:
        y += Dv * u
    if z is not None:
        y *= _silu(z)
    return y, hL


def _head_case(rng, Bsz, nheads, P, L, N, shared):
    D = nheads * P
    c = dict(u=rng.standard_normal((Bsz, D, L)), delta=0.5 * rng.standard_normal((Bsz, D, L)),
             z=rng.standard_normal((Bsz, D, L)), A=-rng.uniform(0.2, 2.0, nheads),
             D=rng.standard_normal(D), delta_bias=rng.uniform(-3, 0.5, D))
    shp = (D, N) if shared else (Bsz, N, L)
    c["B"], c["C"] = rng.standard_normal(shp), rng.standard_normal(shp)
    return c


def _bc_rows(c, b, d, L):
    if c["B"].ndim == 2:                     # time-invariant: row d at every position
        return np.tile(c["B"][d], (L, 1)), np.tile(c["C"][d], (L, 1))
    return c["B"][b].T, c["C"][b].T


@pytest.mark.parametrize("N,shared", [(4, False), (4, True), (64, False), (16, True)])
def test_scalar_A_per_head_equals_ssd_dual_form(N, shared):
    """A one scalar per head: every channel of head h decays all its states with A_h."""
    rng = np.random.default_rng(81)
    Bsz, nheads, P, L = 2, 3, 2, 11
    c = _head_case(rng, Bsz, nheads, P, L, N, shared)
    y, hf = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                                  c["delta_bias"], True, return_final_state=True)
    dl = _softplus(c["delta"] + c["delta_bias"][None, :, None])
    for b in range(Bsz):
        for d in range(nheads * P):
            Bt, Ct = _bc_rows(c, b, d, L)
            A_dn = np.full(N, c["A"][d // P])
            yd, hd = _dual_form(c["u"][b, d], dl[b, d], A_dn, Bt, Ct, c["D"][d], c["z"][b, d])
            np.testing.assert_allclose(y[b, d], yd, rtol=1e-10, atol=1e-12)
            np.testing.assert_allclose(hf[b, d], hd, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("N", [8, 128])
def test_per_state_A_equals_dual_form(N):
    """The general diagonal A (dim, N), variable B/C, at d_state up to 128."""
    rng = np.random.default_rng(82)
    c = _rand_case(rng, B=1, D=2, L=9, N=N)
    y, hf = oracle.selective_scan(c["u"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                                  c["delta_bias"], True, return_final_state=True)
    dl = _softplus(c["delta"] + c["delta_bias"][None, :, None])
    for d in range(2):
        yd, hd = _dual_form(c["u"][0, d], dl[0, d], c["A"][d], c["B"][0].T, c["C"][0].T,
                            c["D"][d], c["z"][0, d])
        np.testing.assert_allclose(y[0, d], yd, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(hf[0, d], hd, rtol=1e-10, atol=1e-12)


def test_time_invariant_BC_constant_inputs_closed_form():
    """Constant delta and u with B, C fixed per channel (the LTI case): each state is a
    geometric series, h_t = delta u B[d, n] (1 - a^(t+1)) / (1 - a), a = exp(delta A)."""
    rng = np.random.default_rng(83)
    Dm, L, N = 3, 12, 5
    A = -rng.uniform(0.1, 1.5, (Dm, N))
    Bs, Cs = rng.standard_normal((Dm, N)), rng.standard_normal((Dm, N))
    dl, uval = 0.37, 0.8
    u = np.full((1, Dm, L), uval)
    delta = np.full((1, Dm, L), dl)
    Dv = rng.standard_normal(Dm)
    y, hf = oracle.selective_scan(u, delta, A, Bs, Cs, Dv, None, None, False,
                                  return_final_state=True)
    t = np.arange(L)
    for d in range(Dm):
        a = np.exp(dl * A[d])                                    # (N,)
        h = dl * uval * Bs[d][None, :] * (1 - a[None, :] ** (t[:, None] + 1)) / (1 - a[None, :])
        np.testing.assert_allclose(y[0, d], h @ Cs[d] + Dv[d] * uval, rtol=1e-12)
        np.testing.assert_allclose(hf[0, d], h[-1], rtol=1e-12)

