"""Seeded synthetic inputs for the selective-scan workloads.

This module only draws numbers. It holds none of the scan's arithmetic, so the
CUDA path and the CPU oracle can both take their inputs from here without
sharing any of the method.

Every tensor comes from its own stream, ``SeedSequence([seed, tensor_id])``, so
adding a tensor never shifts the values of another. Activations that the GPU
receives in bf16 are rounded to bf16 (round to nearest, ties to even) here, and
the rounded values are what both sides consume.

Value recipe (the Mamba block's initialisation as the pyshine.com "Mamba" tour
describes it, section "Why You Need This": dt bias placed so that softplus of
it lies in [dt_min, dt_max]; A from the S4D-real initialisation, kept in fp32):

* u (or the pre-conv x), z, B, C ~ N(0, 1)
* A[d, n] = -(n + 1); A given per head (Mamba-2 style): A[h] = -U(1, 16)
* time-invariant B, C: fp32 (dim, dstate) ~ N(0, 1)
* D ~ N(0, 1)
* dt_bias[d] = log(expm1(y)), y = exp(U(ln 1e-3, ln 0.1)) per channel
* dt_raw ~ N(0, 0.5**2)
* conv weight ~ N(0, 0.5**2), conv bias 0
* decode: SSM state ~ N(0, 1) fp32; conv state ~ N(0, 1) in the activation dtype
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# One stream id per tensor role.
TID = {
    "u": 1, "delta": 2, "z": 3, "B": 4, "C": 5, "D": 6, "delta_bias": 7,
    "conv_w": 8, "D_rev": 9, "delta_bias_rev": 10, "state": 11, "conv_state": 12,
    "dec_x": 13, "dec_dt": 14, "dec_z": 15, "dec_B": 16, "dec_C": 17,
    "A_rev": 18, "lengths": 19, "A_heads": 20, "A_heads_rev": 21, "B_fixed": 22,
    "C_fixed": 23,
}


def rng(seed: int, tensor_id: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor_id])))


def round_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 -> nearest bf16 value (ties to even), returned as fp32."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    r = (b + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Bit patterns (uint16) of values that are already bf16-representable."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    if np.any(b & np.uint32(0xFFFF)):
        raise ValueError("values are not bf16-representable; round them first")
    return (b >> np.uint32(16)).astype(np.uint16)


def normal(seed: int, role: str, shape, std: float = 1.0) -> np.ndarray:
    g = rng(seed, TID[role])
    x = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def s4d_real_A(dim: int, dstate: int) -> np.ndarray:
    return np.tile(-np.arange(1, dstate + 1, dtype=np.float32), (dim, 1))


def heads_A(seed: int, role: str, nheads: int) -> np.ndarray:
    """One negative scalar per head, -U(1, 16)."""
    return (-rng(seed, TID[role]).uniform(1.0, 16.0, size=nheads)).astype(np.float32)


def dt_bias(seed: int, role: str, dim: int, dt_min=1e-3, dt_max=0.1) -> np.ndarray:
    g = rng(seed, TID[role])
    y = np.exp(g.uniform(np.log(dt_min), np.log(dt_max), size=dim))
    return np.log(np.expm1(y)).astype(np.float32)


@dataclass
class Workload:
    """One selective-scan workload (shapes and switches)."""
    name: str
    batch: int
    dim: int
    seqlen: int
    dstate: int = 16
    dtype: str = "f32"          # "f32" or "bf16" for u/delta/z/B/C/out
    conv_width: int = 0         # 0 = no fused conv
    bidirectional: bool = False
    final_state: bool = False
    steps: int = 0              # decode steps (decode workload only)
    extra: dict = field(default_factory=dict)

    @property
    def elems(self) -> int:
        return self.batch * self.dim * max(self.seqlen, 1)


WORKLOADS = {
    "tiny": Workload("tiny fp32 scan B1 D64 L256 N16", 1, 64, 256, 16, "f32"),
    "m130": Workload("Mamba-130M layer B8 D1536 L2048 N16 bf16 + conv4", 8, 1536, 2048, 16,
                     "bf16", conv_width=4),
    "long": Workload("Mamba-2.8B long B1 D5120 L65536 N16 bf16 + final state", 1, 5120, 65536,
                     16, "bf16", final_state=True),
    "bidir": Workload("bidirectional B16 D768 L1024 N16 fp32", 16, 768, 1024, 16, "f32",
                      bidirectional=True),
    "decode": Workload("decode B256 D5120 N16 bf16 x64 steps", 256, 5120, 1, 16, "bf16",
                       conv_width=4, steps=64),
    "decode_h128": Workload("decode B256 D1536 (24 heads x 64) N128 bf16 x64 steps: A one scalar "
                            "per head (Mamba-2-130M shape)", 256, 1536, 1, 128, "bf16",
                            conv_width=4, steps=64, extra={"a_heads": 24}),
    "conv": Workload("causal conv1d + SiLU B8 D1536 L2048 bf16 width 4", 8, 1536, 2048, 16,
                     "bf16", conv_width=4, extra={"conv_only": True}),
    "m130_cl": Workload("Mamba-130M layer in the block's layout B8 L2048 D1536 N16 bf16 + conv4: "
                        "x, z halves of one (B, L, 2D) in_proj output; B, C columns of one "
                        "(B, L, 48 + 2N) x_proj output", 8, 1536, 2048, 16, "bf16", conv_width=4,
                        extra={"channel_last": True, "dt_rank": 48}),
    "heads128": Workload("Mamba-2-130M-shaped scan B8 L2048 D1536 (24 heads x 64) N128 bf16 + "
                         "conv4: A one scalar per head", 8, 1536, 2048, 128, "bf16", conv_width=4,
                         extra={"a_heads": 24}),
    "varlen": Workload("packed sequences B1 D1536 L32768 N16 bf16 + conv4, lengths "
                       "log-uniform in [64, 4096]", 1, 1536, 32768, 16, "bf16", conv_width=4,
                       final_state=True, extra={"packed": (64, 4096)}),
}


def packed_lengths(total: int, lo: int, hi: int, seed: int = 0) -> np.ndarray:
    """Sequence lengths for packed-sequence workloads: log-uniform in [lo, hi], drawn
    from their own stream until they cover `total`; the last one is cut to fit."""
    g = rng(seed, TID["lengths"])
    lens = []
    while sum(lens) < total:
        lens.append(int(round(np.exp(g.uniform(np.log(lo), np.log(hi))))))
    lens[-1] -= sum(lens) - total
    return np.array([n for n in lens if n > 0], dtype=np.int64)


def _act(x: np.ndarray, dtype: str) -> np.ndarray:
    return round_bf16(x) if dtype == "bf16" else x.astype(np.float32)


def scan_inputs(batch: int, dim: int, seqlen: int, dstate: int = 16, dtype: str = "f32",
                conv_width: int = 0, bidirectional: bool = False, seed: int = 0,
                a_heads: int = 0, bc_shared: bool = False) -> dict:
    """All inputs of one scan call as fp32 numpy arrays (activations bf16-rounded if bf16).

    Layouts: u, delta, z (batch, dim, seqlen); B, C (batch, dstate, seqlen), or fp32
    (dim, dstate) with ``bc_shared``; A (dim, dstate), or (a_heads,) with ``a_heads``;
    D, delta_bias (dim); conv_w (dim, conv_width); conv_b (dim).
    """
    shp = (batch, dim, seqlen)
    out = {
        "u": _act(normal(seed, "u", shp), dtype),
        "delta": _act(normal(seed, "delta", shp, 0.5), dtype),
        "z": _act(normal(seed, "z", shp), dtype),
        "B": _act(normal(seed, "B", (batch, dstate, seqlen)), dtype),
        "C": _act(normal(seed, "C", (batch, dstate, seqlen)), dtype),
        "A": s4d_real_A(dim, dstate),
        "D": normal(seed, "D", (dim,)),
        "delta_bias": dt_bias(seed, "delta_bias", dim),
    }
    if conv_width:
        out["conv_w"] = normal(seed, "conv_w", (dim, conv_width), 0.5)
        out["conv_b"] = np.zeros(dim, dtype=np.float32)
    if bidirectional:
        out["A_rev"] = s4d_real_A(dim, dstate)
        out["D_rev"] = normal(seed, "D_rev", (dim,))
        out["delta_bias_rev"] = dt_bias(seed, "delta_bias_rev", dim)
    if a_heads:
        out["A"] = heads_A(seed, "A_heads", a_heads)
        if bidirectional:
            out["A_rev"] = heads_A(seed, "A_heads_rev", a_heads)
    if bc_shared:
        out["B"] = normal(seed, "B_fixed", (dim, dstate))
        out["C"] = normal(seed, "C_fixed", (dim, dstate))
    return out


def decode_inputs(batch: int, dim: int, dstate: int = 16, steps: int = 1, conv_width: int = 4,
                  dtype: str = "bf16", seed: int = 0, a_heads: int = 0) -> dict:
    """Inputs of ``steps`` successive single-token updates.

    Layouts: state (batch, dim, dstate) fp32; conv_state (batch, dim, conv_width), newest
    last; per-step x, dt, z (steps, batch, dim); B_t, C_t (steps, batch, dstate);
    A (dim, dstate), or (a_heads,) with ``a_heads``; D, dt_bias, conv_b (dim);
    conv_w (dim, conv_width).
    """
    out = {
        "state": normal(seed, "state", (batch, dim, dstate)),
        "conv_state": _act(normal(seed, "conv_state", (batch, dim, conv_width)), dtype),
        "x": _act(normal(seed, "dec_x", (steps, batch, dim)), dtype),
        "dt": _act(normal(seed, "dec_dt", (steps, batch, dim), 0.5), dtype),
        "z": _act(normal(seed, "dec_z", (steps, batch, dim)), dtype),
        "B": _act(normal(seed, "dec_B", (steps, batch, dstate)), dtype),
        "C": _act(normal(seed, "dec_C", (steps, batch, dstate)), dtype),
        "A": s4d_real_A(dim, dstate),
        "D": normal(seed, "D", (dim,)),
        "dt_bias": dt_bias(seed, "delta_bias", dim),
        "conv_w": normal(seed, "conv_w", (dim, conv_width), 0.5),
        "conv_b": np.zeros(dim, dtype=np.float32),
    }
    if a_heads:
        out["A"] = heads_A(seed, "A_heads", a_heads)
    return out
