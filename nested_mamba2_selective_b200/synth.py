"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module draws random numbers and rounds them to the storage precision; it
holds none of the block's forward arithmetic.  Every array it returns is float32
whose values are exactly representable in the requested storage type, so the
same values can be handed to the GPU (as bf16 or fp32) and to the fp64 oracle.

Recipe (the pages give model sizes but no initialisation; these are the draws
used everywhere in this repository):
  u ~ N(0, 1);  W_in, W_out, conv_w, conv_b ~ N(0, 0.02);  norm_w = 1 + N(0, 0.02)
  A = -exp(U(log 1, log 16));  dt0 = exp(U(log 1e-3, log 1e-1));
  dt_bias = dt0 + log(-expm1(-dt0))   (so that softplus(dt_bias) = dt0)
  D ~ N(0, 1)
  standalone scan inputs: x, B, C ~ N(0, 1); dt ~ exp(U(log 1e-3, log 1e-1)).
Storage: W_in, conv_w, conv_b, norm_w, W_out, u, x, B, C in the workload dtype;
dt_bias, A, D, dt always fp32.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


def bf16_bits(a) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even); return the raw bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32).astype(np.uint64)
    bits = (bits + 0x7FFF + ((bits >> 16) & 1)) >> 16
    return bits.astype(np.uint16)


def bf16_value(bits: np.ndarray) -> np.ndarray:
    """float32 array holding the values of the given bfloat16 bit patterns."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def round_to(a, dtype: str) -> np.ndarray:
    """Values of ``a`` rounded to the storage type ('bf16' or 'f32'), as float32."""
    if dtype == "bf16":
        return bf16_value(bf16_bits(a))
    if dtype == "f32":
        return np.ascontiguousarray(a, dtype=np.float32)
    raise ValueError(dtype)


@dataclass(frozen=True)
class Workload:
    """One named workload: model sizes, batch shape, widths and storage type."""
    name: str
    kind: str            # 'block', 'ssd', 'stack', 'decode'
    dtype: str           # 'f32' or 'bf16'
    batch: int
    seqlen: int
    d_model: int = 0
    d_inner: int = 0
    d_head: int = 64
    d_state: int = 128
    ngroups: int = 1
    d_conv: int = 4
    chunk: int = 256
    nheads: int = 0      # standalone scan: number of heads in the tensors
    nlayers: int = 1
    steps: int = 0
    widths: tuple = field(default_factory=tuple)
    seed: int = 0


WORKLOADS = {
    w.name: w for w in (
        Workload("block_tiny_f32", "block", "f32", batch=1, seqlen=64, d_model=64, d_inner=128, d_head=32,
                 d_state=16, chunk=16, widths=(64, 32, 16), seed=1000),
        Workload("ssd_b4_L8192_h24", "ssd", "bf16", batch=4, seqlen=8192, d_head=64, d_state=128, chunk=256,
                 nheads=24, widths=(24, 12), seed=1001),
        Workload("block_130m_b8_L2048", "block", "bf16", batch=8, seqlen=2048, d_model=768, d_inner=1536,
                 chunk=256, widths=(768, 384, 192, 96), seed=1002),
        Workload("stack48_1p4b_b4_L4096", "stack", "bf16", batch=4, seqlen=4096, d_model=2048, d_inner=4096,
                 chunk=256, nlayers=48, widths=(2048, 1024, 512, 256), seed=1003),
        Workload("decode_b256_1p4b", "decode", "bf16", batch=256, seqlen=1, d_model=2048, d_inner=4096,
                 steps=1000, widths=(2048, 1024, 512), seed=1004),
    )
}


def _normal(rng, shape, std=1.0, mean=0.0):
    return (rng.standard_normal(shape, dtype=np.float32) * np.float32(std) + np.float32(mean))


def _log_uniform(rng, shape, lo, hi):
    return np.exp(rng.uniform(np.log(lo), np.log(hi), size=shape)).astype(np.float32)


def block_params(d_model, d_inner, d_head, d_state, ngroups=1, d_conv=4, dtype="bf16", seed=0):
    """Full-width parameters of one block as float32 arrays holding storage-exact values.

    Keys: W_in (2E+2GN+H, d_model) rows z|x|B|C|dt, conv_w (E+2GN, d_conv), conv_b (E+2GN),
    dt_bias (H), A (H), D (H), norm_w (E), W_out (d_model, E)."""
    E, GN = d_inner, ngroups * d_state
    H = E // d_head
    rng = np.random.Generator(np.random.PCG64(seed))
    p = {}
    p["W_in"] = round_to(_normal(rng, (2 * E + 2 * GN + H, d_model), 0.02), dtype)
    p["conv_w"] = round_to(_normal(rng, (E + 2 * GN, d_conv), 0.02), dtype)
    p["conv_b"] = round_to(_normal(rng, (E + 2 * GN,), 0.02), dtype)
    dt0 = _log_uniform(rng, (H,), 1e-3, 1e-1).astype(np.float64)
    p["dt_bias"] = (dt0 + np.log(-np.expm1(-dt0))).astype(np.float32)
    p["A"] = (-np.exp(rng.uniform(np.log(1.0), np.log(16.0), size=(H,)))).astype(np.float32)
    p["D"] = _normal(rng, (H,), 1.0)
    p["norm_w"] = round_to(_normal(rng, (E,), 0.02, 1.0), dtype)
    p["W_out"] = round_to(_normal(rng, (d_model, E), 0.02), dtype)
    return p


def activations(shape, dtype="bf16", seed=0, std=1.0):
    """u ~ N(0, std^2) rounded to the storage type."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return round_to(_normal(rng, shape, std), dtype)


def ssd_inputs(batch, L, h, P, N, G=1, dtype="bf16", seed=0):
    """Standalone scan inputs: x (b,L,h,P), dt (b,L,h) post-softplus, A (h), B, C (b,L,G,N), D (h)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = round_to(_normal(rng, (batch, L, h, P)), dtype)
    B = round_to(_normal(rng, (batch, L, G, N)), dtype)
    C = round_to(_normal(rng, (batch, L, G, N)), dtype)
    dt = _log_uniform(rng, (batch, L, h), 1e-3, 1e-1)
    A = (-np.exp(rng.uniform(np.log(1.0), np.log(16.0), size=(h,)))).astype(np.float32)
    D = _normal(rng, (h,), 1.0)
    return dict(x=x, dt=dt, A=A, B=B, C=C, D=D)


def long_memory(inputs: dict) -> dict:
    """Test-only variant of the scan inputs with slow decay (dt = 1e-3, A = -1), so that the
    state carried across chunk and segment boundaries stays visible in the output."""
    out = dict(inputs)
    out["dt"] = np.full_like(inputs["dt"], 1e-3)
    out["A"] = np.full_like(inputs["A"], -1.0)
    return out


def states(batch, H, P, N, conv_rows, d_conv, dtype="bf16", seed=0):
    """Prefilled recurrent state ~ N(0, 1): ssm (b,H,P,N) fp32 and conv (b, rows, d_conv-1) in dtype."""
    rng = np.random.Generator(np.random.PCG64(seed))
    ssm = _normal(rng, (batch, H, P, N))
    conv = round_to(_normal(rng, (batch, conv_rows, d_conv - 1)), dtype)
    return ssm, conv
