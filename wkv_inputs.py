"""Seeded synthetic inputs for the WKV operator.

This module only draws random numbers and rounds them to the storage dtype. It holds
none of the operator's arithmetic and imports neither the CUDA package nor the oracle,
so both sides (and the benchmark) can take their inputs from here.

Recipe (all draws from ``numpy.random.Generator(PCG64(seed))``, in this order):

* log w ~ U(lo, hi) per channel, w = exp(log w)  (w > 0, the decay rate);
* u ~ U(-bu, bu) per channel (the bonus of the current token);
* k ~ N(0, k_std), v ~ N(0, 1), r ~ N(0, 1) over (B, T, C), C fastest;
* optionally dy ~ N(0, 1) over (B, T, C) (upstream gradient);
* optionally a Bernoulli(spike_frac) mask over (B, T, C) whose entries of k are set
  to ``spike_value`` (overflow stress).

The per-channel parameters are drawn in float64 and rounded to float32. The (B, T, C)
tensors are drawn as float32 standard normals (NumPy's float32 ziggurat, about five
times faster than float64 draws, which matters at 10^8 elements) and scaled by k_std in
float32; for bf16 storage the float32 values are rounded to bf16 (round to nearest even).
The arrays handed out are the *stored* values: float32 arrays, or, for bf16, the
float32 arrays holding exactly the bf16 values plus the raw uint16 bit patterns.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


def round_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even. NaN-free input."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    r = u >> np.uint32(16)
    r &= np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u
    r >>= np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> the exactly equal float32 values."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class WkvInputs:
    """One seeded problem. Every float array is float32 and holds the stored values."""

    B: int
    T: int
    C: int
    dtype: str                      # "f32" or "bf16": storage dtype of k, v, r, y
    w: np.ndarray                   # [C] float32, > 0
    u: np.ndarray                   # [C] float32
    k: np.ndarray                   # [B, T, C]
    v: np.ndarray
    r: np.ndarray
    dy: np.ndarray | None = None    # [B, T, C] float32 (always fp32)
    bits: dict = field(default_factory=dict)  # bf16 only: name -> uint16 [B, T, C]


def _store(x32: np.ndarray, dtype: str):
    if dtype == "f32":
        return x32, None
    if dtype == "bf16":
        b = round_to_bf16_bits(x32)
        return bf16_bits_to_f32(b), b
    raise ValueError(f"unknown dtype {dtype!r}")


def make_inputs(B: int, T: int, C: int, seed: int = 0, *, dtype: str = "f32",
                logw_range=(-5.0, 1.0), u_bound: float = 1.0, k_std: float = 1.0,
                spike_frac: float = 0.0, spike_value: float = 60.0,
                with_dy: bool = False) -> WkvInputs:
    """Draw one problem following the recipe in the module docstring."""
    g = np.random.Generator(np.random.PCG64(seed))
    logw = g.uniform(logw_range[0], logw_range[1], size=C)
    w = np.exp(logw).astype(np.float32)
    u = g.uniform(-u_bound, u_bound, size=C).astype(np.float32)
    shape = (B, T, C)
    f32 = np.float32
    k32 = g.standard_normal(size=shape, dtype=f32)
    if k_std != 1.0:
        k32 *= f32(k_std)
    v32 = g.standard_normal(size=shape, dtype=f32)
    r32 = g.standard_normal(size=shape, dtype=f32)
    dy = g.standard_normal(size=shape, dtype=f32) if with_dy else None
    if spike_frac > 0.0:
        mask = g.random(size=shape, dtype=f32) < f32(spike_frac)
        k32[mask] = f32(spike_value)
        del mask
    out = WkvInputs(B, T, C, dtype, w, u, None, None, None, dy)
    for name, x32 in (("k", k32), ("v", v32), ("r", r32)):
        x, bits = _store(x32, dtype)
        setattr(out, name, x)
        if bits is not None:
            out.bits[name] = bits
    return out


# The five workloads the operator is measured and checked on.
def tiny_forward(seed: int = 0) -> WkvInputs:
    """fp32 forward, B=1, T=64, C=128."""
    return make_inputs(1, 64, 128, seed)


def training_shape(seed: int = 0, B: int = 16, T: int = 1024, C: int = 768) -> WkvInputs:
    """fp32 forward + backward at the 169M-model training shape B=16, T=1024, C=768."""
    return make_inputs(B, T, C, seed, with_dy=True)


def long_bf16(seed: int = 0, B: int = 8, T: int = 4096, C: int = 4096) -> WkvInputs:
    """bf16 forward at the 7B-model shape B=8, T=4096, C=4096 with k spikes of +60."""
    return make_inputs(B, T, C, seed, dtype="bf16", logw_range=(-6.0, 2.0), u_bound=2.0,
                       k_std=3.0, spike_frac=1e-3, spike_value=60.0)


def long_context(seed: int = 0, B: int = 1, T: int = 32768, C: int = 4096,
                 stress: bool = False) -> WkvInputs:
    """fp32 forward over one long sequence B=1, T=32768, C=4096.

    ``stress=True`` swaps in the bf16 workload's distributions (k ~ N(0,3) with spikes).
    """
    if stress:
        return make_inputs(B, T, C, seed, logw_range=(-6.0, 2.0), u_bound=2.0, k_std=3.0,
                           spike_frac=1e-3, spike_value=60.0)
    return make_inputs(B, T, C, seed)


@dataclass
class DecodeInputs:
    """Batched decode: N sequences x L layers x C channels, chained over steps."""

    N: int
    L: int
    C: int
    w: np.ndarray   # [L, C] float32
    u: np.ndarray   # [L, C] float32
    a: np.ndarray   # [N, L, C] float32 initial state numerator (scaled)
    b: np.ndarray   # [N, L, C] float32 initial state denominator (scaled), > 0
    p: np.ndarray   # [N, L, C] float32 initial state log-scale (natural log)
    seed: int

    def step(self, s: int):
        """k, v, r for step s, each [N, L, C] float32; step s has its own stream
        (PCG64 seeded with [seed, 1 + s]) and draws float32 normals directly, so that the
        64 chained steps of the full workload can be generated quickly."""
        g = np.random.Generator(np.random.PCG64([self.seed, 1 + s]))
        shape = (self.N, self.L, self.C)
        return tuple(g.standard_normal(size=shape, dtype=np.float32) for _ in range(3))


def decode_batch(seed: int = 0, N: int = 256, L: int = 32, C: int = 4096) -> DecodeInputs:
    """Decode workload: state (a,b,p) ~ (N(0,1), U(0.5,2), N(0,1)), w = exp(U(-5,1)),
    u ~ U(-1,1) per (layer, channel); per-step k, v, r ~ N(0,1)."""
    g = np.random.Generator(np.random.PCG64(seed))
    shape = (N, L, C)
    a = g.standard_normal(size=shape).astype(np.float32)
    b = g.uniform(0.5, 2.0, size=shape).astype(np.float32)
    p = g.standard_normal(size=shape).astype(np.float32)
    w = np.exp(g.uniform(-5.0, 1.0, size=(L, C))).astype(np.float32)
    u = g.uniform(-1.0, 1.0, size=(L, C)).astype(np.float32)
    return DecodeInputs(N, L, C, w, u, a, b, p, seed)


def sample_channels(B: int, C: int, n: int, seed: int = 12345):
    """n distinct seeded (b, c) pairs, for checks that look at whole time series."""
    g = np.random.Generator(np.random.PCG64(seed))
    n = min(n, B * C)
    flat = g.choice(B * C, size=n, replace=False)
    return [(int(f // C), int(f % C)) for f in np.sort(flat)]


@dataclass
class Wkv7Inputs:
    """One seeded RWKV-7 problem: (B, T, H, N) float32 tensors and an initial state."""

    B: int
    T: int
    H: int
    N: int
    r: np.ndarray
    w: np.ndarray      # decay factor in (0.5, 1]
    k: np.ndarray
    v: np.ndarray
    a: np.ndarray      # -kappa^ (unit per head and token)
    b: np.ndarray      # kappa^ * alpha, alpha ~ U(0, 1) per channel
    S0: np.ndarray     # (B, H, N, N)


def rwkv7_inputs(B: int, T: int, H: int, N: int = 64, seed: int = 0) -> Wkv7Inputs:
    """RWKV-7 recurrence inputs (research report, section 1.3.3: decay w_t, in-context
    learning vectors a_t, b_t). Draw order from PCG64(seed): r, k, v ~ N(0, 1); w = exp(-x)
    with x ~ U(0, 0.7); kappa ~ N(0, 1) normalised per (b, t, h) to kappa^; alpha ~ U(0, 1);
    a = -kappa^, b = kappa^ alpha (the delta rule's removal of the old value along kappa^,
    so the transition diag(w) + a^T b stays contracting); S0 ~ N(0, 0.1). All float32."""
    g = np.random.Generator(np.random.PCG64(seed))
    shape = (B, T, H, N)

    def normal(scale=1.0):
        x = g.standard_normal(shape, dtype=np.float32)
        return x if scale == 1.0 else x * np.float32(scale)

    r, k, v = normal(), normal(), normal()
    w = np.exp(-g.uniform(0.0, 0.7, size=shape)).astype(np.float32)
    kap = normal()
    kap /= np.linalg.norm(kap, axis=-1, keepdims=True)
    alpha = g.uniform(0.0, 1.0, size=shape).astype(np.float32)
    a = -kap
    b = (kap * alpha).astype(np.float32)
    S0 = g.standard_normal((B, H, N, N), dtype=np.float32) * np.float32(0.1)
    return Wkv7Inputs(B, T, H, N, r, w, k, v, a.astype(np.float32), b, S0)
