"""Seeded synthetic inputs and the named workloads.

This module holds no arithmetic of the operator itself: it only draws the
inputs.  Both the CUDA path and the CPU oracle are fed from here.

Distributions (2Mamba2Furious, Algorithm 2 "Mamba-2 Setup"):
  * Q, K, V = SiLU(N(0, 1)) -- the Algorithm 3 activation applied to a
    standard normal stand-in for the projected, convolved activations;
  * dt_P ~ N(0, 1);
  * A_log = log(U[1, 16]) per head;
  * dt_bias = softplus^-1(dt_init) = dt_init + log(1 - exp(-dt_init)) with
    dt_init = exp(U[log 1e-3, log 1e-1]) per head;
  * D = ones(H * d_h).

Random numbers come from numpy's PCG64 generator seeded with ``seed`` and are
drawn in the fixed order q, k, v, dt_p, A_log, dt_bias.  For bf16 workloads
q, k and v are rounded to bf16 with round-to-nearest-even; the float32 arrays
returned hold exactly the rounded values, and ``*_bits`` hold the bf16 bit
patterns the device receives.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

DT_MIN = 1e-3
DT_MAX = 1e-1


@dataclasses.dataclass(frozen=True)
class Workload:
    """One operator invocation shape: [B, H, N, d] activations, chunk length,
    order (1 = plain scores, 2 = squared scores), normaliser and D-residual."""
    name: str
    B: int
    H: int
    N: int
    d: int
    chunk: int
    order: int
    normalize: bool
    residual: bool
    dtype: str  # "f32" or "bf16"

    @property
    def tokens(self) -> int:
        return self.B * self.N

    @property
    def token_heads(self) -> int:
        return self.B * self.H * self.N


# The five workloads the operator is specified on (names say what they are).
WORKLOADS: Dict[str, Workload] = {w.name: w for w in [
    Workload("order1-fp32-B1H2N256d16-c64", 1, 2, 256, 16, 64, 1, False, True, "f32"),
    Workload("order1-bf16-B4H16N2048d64-c128", 4, 16, 2048, 64, 128, 1, False, True, "bf16"),
    Workload("order2-bf16-B4H16N4096d32-c64", 4, 16, 4096, 32, 64, 2, True, False, "bf16"),
    Workload("order1-bf16-B1H32N65536d64-c256", 1, 32, 65536, 64, 256, 1, False, False, "bf16"),
    Workload("order2-bf16-B2H8N16384d64-c64", 2, 8, 16384, 64, 64, 2, True, True, "bf16"),
]}
WORKLOAD_ORDER = list(WORKLOADS.keys())
SMALL = WORKLOAD_ORDER[0]   # the order-1 fp32 case the oracle finishes instantly
HEADLINE = WORKLOAD_ORDER[1]  # the H=16, d_h=64, N=2048 order-1 bf16 case


def bf16_round_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> the float32 values they encode."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _silu_normal(rng: np.random.Generator, shape) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    # SiLU(x) = x * sigmoid(x); in place to keep peak memory at one buffer.
    e = np.exp(-x)
    e += np.float32(1.0)
    np.divide(x, e, out=x)
    del e
    return x


def make_inputs(B: int, H: int, N: int, d: int, dtype: str = "bf16", seed: int = 0,
                residual: bool = True) -> Dict[str, Optional[np.ndarray]]:
    """Draw one seeded input set.

    Returns a dict with float32 arrays q, k, v [B, H, N, d] (bf16-exact when
    dtype is "bf16"), dt_p [B, H, N], A_log [H], dt_bias [H], D [H*d] (None
    when ``residual`` is False), and for bf16 the uint16 arrays q_bits,
    k_bits, v_bits."""
    if dtype not in ("f32", "bf16"):
        raise ValueError("dtype must be 'f32' or 'bf16'")
    rng = np.random.Generator(np.random.PCG64(seed))
    shape = (B, H, N, d)
    out: Dict[str, Optional[np.ndarray]] = {}
    for name in ("q", "k", "v"):
        x = _silu_normal(rng, shape)
        if dtype == "bf16":
            bits = bf16_round_bits(x)
            out[name + "_bits"] = bits
            x = bf16_bits_to_f32(bits)
        out[name] = x
    out["dt_p"] = rng.standard_normal(size=(B, H, N), dtype=np.float32)
    out["A_log"] = np.log(rng.uniform(1.0, 16.0, size=H)).astype(np.float32)
    dt_init = np.exp(rng.uniform(np.log(DT_MIN), np.log(DT_MAX), size=H))
    # inverse of softplus: y + log(1 - exp(-y))
    out["dt_bias"] = (dt_init + np.log(-np.expm1(-dt_init))).astype(np.float32)
    out["D"] = np.ones(H * d, dtype=np.float32) if residual else None
    return out


def make_workload_inputs(w: Workload, seed: int = 0, residual: Optional[bool] = None):
    """make_inputs for a named workload (residual defaults to the workload's)."""
    res = w.residual if residual is None else residual
    return make_inputs(w.B, w.H, w.N, w.d, w.dtype, seed, res)


def make_log_decay(B: int, H: int, N: int, seed: int = 0, mean: float = -2.0) -> np.ndarray:
    """Per-token log-decays for the Mamba-2S input form (Algorithm 4,
    A = -softplus(h W_A)), with the projection h W_A drawn as N(mean, 1).
    Returns float32 [B, H, N], every entry < 0 (mean -0.13 for mean = -2)."""
    rng = np.random.Generator(np.random.PCG64(seed + 1000))
    z = rng.standard_normal(size=(B, H, N)) + mean
    return (-(np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z))))).astype(np.float32)
