"""The oracle's recurrence readings against vLLM's Mamba kernels (GPU, fp32).

The pages validate against the implementations by Tri Dao and vLLM for agreement
within floating-point tolerance (qwerky.ai "Bringing Blazing-Fast State Space Models
to the Modular MAX Framework", validation paragraphs). vLLM's single-token
``selective_state_update`` and its ``selective_scan_fn`` run here on small fp32 cases,
and the double-precision ORACLE (not this library's kernels) must agree with them.
This fixes, from outside the oracle, the readings the pages leave open: softplus
applied to dt + dt_bias, the bias added without softplus when softplus is off,
dA = exp(delta*A), dBu = delta*B*u, D*u inside the z gate, y = C.h + D*u, and the
final state.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def _rel(got, ref):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref * ref)) + 1e-30
    return float(np.max(np.abs(got - ref) / np.maximum(np.abs(ref), rms)))


def _vllm_ops():
    try:
        from vllm.model_executor.layers.mamba.ops import mamba_ssm
    except Exception as e:                  # pragma: no cover - depends on the image
        pytest.skip(f"vLLM's mamba ops do not import here: {e!r}")
    return mamba_ssm


@pytest.mark.parametrize("softplus,gate", [(True, True), (False, True), (True, False)])
def test_state_update_oracle_matches_vllm(softplus, gate):
    mamba_ssm = _vllm_ops()
    g = np.random.default_rng(7)
    Bsz, D, N = 4, 64, 16
    st = g.standard_normal((Bsz, D, N))
    x, z = g.standard_normal((Bsz, D)), g.standard_normal((Bsz, D))
    dt = 0.5 * g.standard_normal((Bsz, D)) + (0.0 if softplus else 1.0)
    A = -g.uniform(0.5, 8.0, (D, N))
    Bm, Cm = g.standard_normal((Bsz, N)), g.standard_normal((Bsz, N))
    Dv, bias = g.standard_normal(D), g.uniform(-3.0, -1.0, D) if softplus else g.uniform(0, 0.3, D)
    cast = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()
    state = cast(st)
    out = torch.empty(Bsz, D, device="cuda")
    mamba_ssm.selective_state_update(state, cast(x), cast(dt), cast(A), cast(Bm), cast(Cm), cast(Dv),
                                     cast(bias), z=cast(z) if gate else None, dt_softplus=softplus,
                                     out=out)
    torch.cuda.synchronize()
    f32 = lambda a: np.asarray(a, np.float32).astype(np.float64)     # the values vLLM saw
    y, st_new, _ = oracle.state_update(f32(st), None, f32(x), f32(dt), f32(A), f32(Bm), f32(Cm),
                                       f32(Dv), f32(z) if gate else None, f32(bias), softplus)
    assert _rel(out.cpu().numpy(), y) < 1e-4
    assert _rel(state.cpu().numpy(), st_new) < 1e-4


@pytest.mark.parametrize("gate", [True, False])
def test_scan_oracle_matches_vllm(gate):
    mamba_ssm = _vllm_ops()
    g = np.random.default_rng(8)
    Bsz, D, L, N = 2, 32, 96, 16
    u, z = g.standard_normal((Bsz, D, L)), g.standard_normal((Bsz, D, L))
    dt = 0.5 * g.standard_normal((Bsz, D, L))
    A = -np.tile(np.arange(1, N + 1, dtype=np.float64), (D, 1)) * g.uniform(0.5, 1.5, (D, 1))
    Bm, Cm = g.standard_normal((Bsz, N, L)), g.standard_normal((Bsz, N, L))
    Dv, bias = g.standard_normal(D), g.uniform(-4.0, -1.0, D)
    cast = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()
    states = torch.zeros(Bsz, D, N, device="cuda")
    try:
        res = mamba_ssm.selective_scan_fn(cast(u), states, cast(dt), cast(A), cast(Bm), cast(Cm),
                                          cast(Dv), cast(z) if gate else None, cast(bias), True)
    except Exception as e:                  # pragma: no cover - depends on the image
        pytest.skip(f"vLLM's compiled selective_scan_fwd is not usable here: {e!r}")
    torch.cuda.synchronize()
    f32 = lambda a: np.asarray(a, np.float32).astype(np.float64)
    y, h = oracle.selective_scan(f32(u), f32(dt), f32(A), f32(Bm), f32(Cm), f32(Dv),
                                 f32(z) if gate else None, f32(bias), True, False,
                                 return_final_state=True)
    assert _rel(res.cpu().numpy(), y) < 1e-4
    assert _rel(states.cpu().numpy(), h) < 1e-4
