"""The oracle's readings of the conv against vLLM's plain-PyTorch Mamba conv (CPU).

The pages validate their kernels against the implementations by Tri Dao and vLLM
(qwerky.ai "Bringing Blazing-Fast State Space Models to the Modular MAX Framework",
validation paragraphs). vLLM ships PyTorch reference versions of the causal conv for
the prefill (``causal_conv1d_torch``) and the decode step (``causal_conv1d_update_torch``).
Here they fix, from outside the oracle, the readings the pages leave open: the tap
orientation (the last tap meets the newest input), the bias added before SiLU, the
conv history read oldest first before position 0, and the decode window shifting left
with the new input appended on the right. Run in float64; the oracle must agree to
rounding.
"""
import numpy as np
import pytest
import torch

import oracle

vllm_conv = pytest.importorskip("vllm.model_executor.layers.mamba.ops.cpu.causal_conv1d")

W = 4


def _case(seed, D=5, L=13):
    g = np.random.default_rng(seed)
    return (g.standard_normal((D, L)), 0.5 * g.standard_normal((D, W)), 0.3 * g.standard_normal(D),
            g.standard_normal((D, W - 1)))


@pytest.mark.parametrize("with_history", [False, True])
def test_prefill_conv_matches_vllm(with_history):
    """The fused conv + SiLU of a scan, observed through y = D*u (B = 0 keeps h = 0,
    D = 1, no gate), against vLLM's prefill conv with or without an initial conv state."""
    x, w, cb, hist = _case(1)
    D, L = x.shape
    ref_states = torch.zeros(1, D, W - 1, dtype=torch.float64)
    if with_history:
        ref_states[0] = torch.from_numpy(hist)
    got_states = ref_states.clone()
    ref = vllm_conv.causal_conv1d_torch(
        torch.from_numpy(x), torch.from_numpy(w), torch.from_numpy(cb), got_states,
        query_start_loc=torch.tensor([0, L]), cache_indices=torch.tensor([0]),
        has_initial_state=torch.tensor([with_history]), activation="silu").numpy()
    N = 2
    y = oracle.selective_scan(x[None], np.zeros((1, D, L)), -np.ones((D, N)), np.zeros((1, N, L)),
                              np.ones((1, N, L)), np.ones(D), None, None, False, False, w, cb,
                              conv_hist=hist[None] if with_history else None)
    np.testing.assert_allclose(y[0], ref, rtol=1e-12, atol=1e-12)
    # the conv state vLLM hands on (last W-1 inputs) is the tail of the oracle's
    # W-long conv state (history ++ x, oldest first)
    tail = oracle.conv_tail(x[None], W, hist[None] if with_history else None)
    np.testing.assert_allclose(tail[0, :, 1:], got_states[0].numpy(), rtol=0, atol=0)


def test_standalone_conv_matches_vllm():
    x, w, cb, _ = _case(2, D=6, L=21)
    D, L = x.shape
    ref = vllm_conv.causal_conv1d_torch(
        torch.from_numpy(x), torch.from_numpy(w), torch.from_numpy(cb),
        torch.zeros(1, D, W - 1, dtype=torch.float64), query_start_loc=torch.tensor([0, L]),
        cache_indices=torch.tensor([0]), has_initial_state=torch.tensor([False]),
        activation="silu").numpy()
    got = oracle.causal_conv1d(x[None], w, cb, True)
    np.testing.assert_allclose(got[0], ref, rtol=1e-12, atol=1e-12)


def test_decode_conv_step_matches_vllm():
    """One decode step's conv (y = D*xc with a zero state and B = 0) and its window
    shift against vLLM's decode conv update; vLLM keeps the last W-1 inputs, the oracle
    the last W (its window after appending x_t)."""
    g = np.random.default_rng(3)
    Bsz, D, N = 3, 5, 4
    cs = g.standard_normal((Bsz, D, W))
    x = g.standard_normal((Bsz, D))
    w = 0.5 * g.standard_normal((D, W))
    cb = 0.3 * g.standard_normal(D)
    y, _, cs_new = oracle.state_update(np.zeros((Bsz, D, N)), cs, x, np.zeros((Bsz, D)),
                                       -np.ones((D, N)), np.zeros((Bsz, N)), np.ones((Bsz, N)),
                                       np.ones(D), None, None, False, w, cb)
    v_state = torch.from_numpy(cs[:, :, 1:].copy())       # vLLM: the W-1 newest inputs
    ref = vllm_conv.causal_conv1d_update_torch(torch.from_numpy(x)[:, :, None], v_state,
                                               torch.from_numpy(w), torch.from_numpy(cb),
                                               activation="silu")
    np.testing.assert_allclose(y, ref[:, :, 0].numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(cs_new[:, :, 1:], v_state.numpy())
    np.testing.assert_array_equal(cs_new[:, :, :-1], cs[:, :, 1:])
