"""Seeded synthetic inputs for one linear layer: calibration activations X and weights W.

This module only draws random numbers and casts them to the storage types the
quantizer consumes (fp32, or bf16 kept as raw uint16 bit patterns).  It holds
none of the quantization arithmetic, so the CUDA path and the CPU oracle can
both be fed from it without sharing any of the method's code.

Every generator takes ``seed`` and uses ``numpy.random.default_rng(seed)``
(PCG64).  The draw order inside each generator is fixed and written out in
the code, so the same seed gives the same bytes on every machine.

Workload shapes follow the GPTQ tutorial page (freeguideonline "GPTQ" article,
section "阶段一": W is d_out x d_in, X is n x d_in) and the layer
configurations of the benchmark this package is measured on:

* ``tiny``   : d_out=256,   d_in=256,   n=512,  X fp32 N(0,1) with 4 channels x20,
               W N(0, 0.02^2); 4-bit asymmetric, group 128.
* ``attn``   : d_out=4096,  d_in=4096,  n=2048, X bf16 with lognormal(0,1) channel
               std and 0.5% of channels x50; W N(0, 0.02^2) with 0.1% entries x10;
               4-bit asymmetric, group 128.
* ``ffn_up`` : d_out=11008, d_in=4096,  n=2048, X bf16 Student-t(4) scaled by a
               lognormal(0,1) channel std; W N(0, 0.02^2); 3-bit symmetric, group 64.
* ``ffn_down``: d_out=4096, d_in=11008, n=4096, X bf16 with 60% zeros and the rest
               |N(0,1)|; W N(0, 0.015^2) with 0.1% entries x10; 2-bit asymmetric
               group 32, then a 4-bit per-row (group -1) pass on the same H.
* ``stack7b``: 32 blocks x {q,k,v,o 4096x4096; gate,up 11008x4096; down 4096x11008},
               each linear layer with its own 2048-token X drawn like ``attn``.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "QuantSpec",
    "Layer",
    "WORKLOADS",
    "bf16_bits_from_f32",
    "f32_from_bf16_bits",
    "make_layer",
    "stack7b_shapes",
]


@dataclass(frozen=True)
class QuantSpec:
    bits: int = 4
    group_size: int = 128
    sym: bool = False
    block_size: int = 128
    damp_rel: float = 0.01


@dataclass
class Layer:
    """One synthetic layer. ``X_bits`` holds bf16 bit patterns when ``x_dtype == 'bf16'``."""

    name: str
    W: np.ndarray                    # float32 [d_out, d_in]
    X: np.ndarray                    # float32 [n, d_in] (exact values of what the GPU reads)
    x_dtype: str                     # 'f32' or 'bf16'
    X_bits: np.ndarray | None        # uint16 [n, d_in] when bf16, else None
    spec: QuantSpec
    extra_specs: list = field(default_factory=list)

    @property
    def d_out(self) -> int:
        return self.W.shape[0]

    @property
    def d_in(self) -> int:
        return self.W.shape[1]

    @property
    def n(self) -> int:
        return self.X.shape[0]


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """Exact fp32 values of bf16 bit patterns."""
    return (b.astype(np.uint32) << 16).view(np.float32)


def _outlier_entries(rng: np.random.Generator, W: np.ndarray, frac: float, factor: float) -> None:
    count = int(round(frac * W.size))
    if count:
        idx = rng.choice(W.size, size=count, replace=False)
        W.reshape(-1)[idx] *= factor


def _lognormal_channels(rng: np.random.Generator, d_in: int, hot_frac: float, hot_factor: float) -> np.ndarray:
    sigma = np.exp(rng.standard_normal(d_in))
    hot = int(round(hot_frac * d_in))
    if hot:
        sigma[rng.choice(d_in, size=hot, replace=False)] *= hot_factor
    return sigma


def _x_heavy(rng, n, d_in, hot_frac=0.005, hot_factor=50.0):
    sigma = _lognormal_channels(rng, d_in, hot_frac, hot_factor)
    return (rng.standard_normal((n, d_in)) * sigma[None, :]).astype(np.float32)


def _x_student(rng, n, d_in, nu=4.0):
    sigma = _lognormal_channels(rng, d_in, 0.0, 1.0)
    return (rng.standard_t(nu, size=(n, d_in)) * sigma[None, :]).astype(np.float32)


def _x_relu2(rng, n, d_in, zero_frac=0.6):
    mag = np.abs(rng.standard_normal((n, d_in)))
    keep = rng.random((n, d_in)) >= zero_frac
    return (mag * keep).astype(np.float32)


def _finish(name, W, Xf, x_dtype, spec, extra=()):
    if x_dtype == "bf16":
        bits = bf16_bits_from_f32(Xf)
        X = f32_from_bf16_bits(bits)
    else:
        bits = None
        X = np.ascontiguousarray(Xf, dtype=np.float32)
    return Layer(name, np.ascontiguousarray(W, dtype=np.float32), X, x_dtype, bits, spec, list(extra))


def make_tiny(seed: int = 0, d_out: int = 256, d_in: int = 256, n: int = 512) -> Layer:
    """X fp32 N(0,1) with 4 random channels x20; W N(0, 0.02^2). Draw order: X, hot channels, W."""
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((n, d_in)).astype(np.float32)
    hot = rng.choice(d_in, size=min(4, d_in), replace=False)
    X[:, hot] *= 20.0
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float32)
    return _finish("tiny", W, X, "f32", QuantSpec(4, 128, False))


def make_attn(seed: int = 0, d_out: int = 4096, d_in: int = 4096, n: int = 2048,
              spec: QuantSpec | None = None) -> Layer:
    """Draw order: channel sigmas, hot channels, X, W, W outlier positions."""
    rng = np.random.default_rng(seed)
    X = _x_heavy(rng, n, d_in)
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float32)
    _outlier_entries(rng, W, 0.001, 10.0)
    return _finish("attn", W, X, "bf16", spec or QuantSpec(4, 128, False))


def make_ffn_up(seed: int = 0, d_out: int = 11008, d_in: int = 4096, n: int = 2048) -> Layer:
    rng = np.random.default_rng(seed)
    X = _x_student(rng, n, d_in)
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float32)
    return _finish("ffn_up", W, X, "bf16", QuantSpec(3, 64, True))


def make_ffn_down(seed: int = 0, d_out: int = 4096, d_in: int = 11008, n: int = 4096) -> Layer:
    rng = np.random.default_rng(seed)
    X = _x_relu2(rng, n, d_in)
    W = (rng.standard_normal((d_out, d_in)) * 0.015).astype(np.float32)
    _outlier_entries(rng, W, 0.001, 10.0)
    return _finish("ffn_down", W, X, "bf16", QuantSpec(2, 32, False),
                   extra=[QuantSpec(4, -1, False)])


def stack7b_shapes() -> list[tuple[str, int, int]]:
    """(name, d_out, d_in) of the 7 linear layers of one 7B-shaped block."""
    return [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
            ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]


def make_stack_layer(block: int, index: int, base_seed: int = 0, n: int = 2048) -> Layer:
    """Layer ``index`` (0..6) of block ``block``; seed = base_seed*1000 + 7*block + index."""
    name, d_out, d_in = stack7b_shapes()[index]
    rng = np.random.default_rng(base_seed * 1000 + 7 * block + index)
    X = _x_heavy(rng, n, d_in)
    W = (rng.standard_normal((d_out, d_in)) * 0.02).astype(np.float32)
    return _finish(f"stack7b.b{block}.{name}", W, X, "bf16", QuantSpec(4, 128, False))


WORKLOADS = {
    "tiny": make_tiny,
    "attn": make_attn,
    "ffn_up": make_ffn_up,
    "ffn_down": make_ffn_down,
}


def make_layer(name: str, seed: int = 0, **kw) -> Layer:
    return WORKLOADS[name](seed=seed, **kw)
