"""Seeded synthetic inputs for the QLoRA linear layer workloads.

This module is the only code shared by the CPU oracle and the CUDA path.  It
draws random numbers and casts them to the storage dtypes; it holds none of
the method's arithmetic (no quantisation, no dequantisation, no matmul).

Recipe (stated once, used everywhere):
  * bit generator: numpy's Philox-4x32-10 counter-based generator, keyed by
    ``seed = 0x510A2026 + 16 * config_index + tensor_id + 32 * linear_index``
    with tensor ids W0=0, A=1, B=2, X=3, dY=4;
  * values: ``standard_normal`` in float64, multiplied by the tensor's sigma;
  * casts: float64 -> float32 with round-to-nearest-even (numpy ``astype``);
    bf16 tensors are then rounded float32 -> bf16 with round-to-nearest-even
    on the bit pattern and handed out as ``uint16`` bit patterns.

Shapes follow the layer's notation: W0 is d x k, A is r x k, B is d x r,
X is T x k, dY is T x d, all row-major.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Tuple

import numpy as np

BASE_SEED = 0x510A2026
TENSOR_IDS = {"W0": 0, "A": 1, "B": 2, "X": 3, "dY": 4}


def seed_for(config_index: int, tensor: str, linear_index: int = 0) -> int:
    return BASE_SEED + 16 * config_index + TENSOR_IDS[tensor] + 32 * linear_index


def normal_f64(seed: int, shape, sigma: float) -> np.ndarray:
    gen = np.random.Generator(np.random.Philox(key=seed))
    out = gen.standard_normal(size=shape, dtype=np.float64)
    if sigma != 1.0:
        out *= sigma
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even) and return uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    bias = 0x7FFF + ((bits >> 16) & 1)
    return ((bits + bias) >> 16).astype(np.uint16)


def normal_f32(seed: int, shape, sigma: float) -> np.ndarray:
    return normal_f64(seed, shape, sigma).astype(np.float32)


def normal_bf16(seed: int, shape, sigma: float) -> np.ndarray:
    """bf16 bit patterns (uint16) of N(0, sigma^2) samples."""
    return f32_to_bf16_bits(normal_f32(seed, shape, sigma))


@dataclasses.dataclass(frozen=True)
class Linear:
    name: str
    d: int      # output features (rows of W0)
    k: int      # input features (cols of W0)


@dataclasses.dataclass(frozen=True)
class Config:
    index: int                 # 1-based, matches the workload table
    name: str
    linears: Tuple[Linear, ...]
    r: int
    alpha: float
    tokens: Tuple[int, ...]
    sigma_w: float
    sigma_b: float = 0.01
    zero_b_variant: bool = False
    merge: bool = False

    @property
    def s(self) -> float:
        return self.alpha / self.r

    @property
    def sigma_a(self) -> float:
        # "A ~ N(0, 1/r)": the second argument is read as a standard deviation.
        return 1.0 / self.r


CONFIGS: List[Config] = [
    Config(1, "single d=k=256 r=8", (Linear("lin", 256, 256),), r=8, alpha=16.0,
           tokens=(16,), sigma_w=0.02, zero_b_variant=True),
    Config(2, "attention projection 4096x4096 r=8", (Linear("proj", 4096, 4096),), r=8,
           alpha=16.0, tokens=(4096,), sigma_w=0.02),
    Config(3, "MLP up 4096->11008 r=16", (Linear("up", 11008, 4096),), r=16, alpha=32.0,
           tokens=(8192,), sigma_w=0.02, merge=True),
    Config(4, "large MLP 8192->22016 and 22016->8192 r=64",
           (Linear("up", 22016, 8192), Linear("down", 8192, 22016)), r=64, alpha=16.0,
           tokens=(16384,), sigma_w=0.015),
    Config(5, "decoder layer, seven linears r=64",
           (Linear("q", 4096, 4096), Linear("k", 4096, 4096), Linear("v", 4096, 4096),
            Linear("o", 4096, 4096), Linear("gate", 11008, 4096), Linear("up", 11008, 4096),
            Linear("down", 4096, 11008)), r=64, alpha=16.0, tokens=(4096, 16), sigma_w=0.02),
]


def config(index: int) -> Config:
    return CONFIGS[index - 1]


@dataclasses.dataclass
class LayerInputs:
    """Host arrays for one linear of one config (bf16 as uint16 bit patterns)."""
    W0: np.ndarray          # float32 (d, k)
    A: np.ndarray           # bf16 bits (r, k)
    B: np.ndarray           # bf16 bits (d, r)
    X: Optional[np.ndarray]  # bf16 bits (T, k)
    dY: Optional[np.ndarray]  # bf16 bits (T, d)
    d: int
    k: int
    r: int
    T: int
    s: float


def make_layer(cfg: Config, linear_index: int = 0, T: Optional[int] = None,
               zero_b: bool = False, with_acts: bool = True,
               shape_override: Optional[Tuple[int, int, int]] = None) -> LayerInputs:
    """Draw the seeded tensors of one linear.

    ``shape_override`` = (d, k, T) keeps the config's seeds and distributions
    but changes the shapes (used for small parity cases with ragged tails).
    """
    lin = cfg.linears[linear_index]
    d, k = lin.d, lin.k
    T = cfg.tokens[0] if T is None else T
    if shape_override is not None:
        d, k, T = shape_override
    r = cfg.r
    ci = cfg.index
    W0 = normal_f32(seed_for(ci, "W0", linear_index), (d, k), cfg.sigma_w)
    A = normal_bf16(seed_for(ci, "A", linear_index), (r, k), cfg.sigma_a)
    if zero_b:
        B = np.zeros((d, r), dtype=np.uint16)
    else:
        B = normal_bf16(seed_for(ci, "B", linear_index), (d, r), cfg.sigma_b)
    X = dY = None
    if with_acts:
        X = normal_bf16(seed_for(ci, "X", linear_index), (T, k), 1.0)
        dY = normal_bf16(seed_for(ci, "dY", linear_index), (T, d), 1.0)
    return LayerInputs(W0=W0, A=A, B=B, X=X, dY=dY, d=d, k=k, r=r, T=T, s=cfg.s)


def custom_layer(seed: int, d: int, k: int, r: int, T: int, alpha: float,
                 sigma_w: float = 0.02, sigma_b: float = 0.01,
                 zero_b: bool = False) -> LayerInputs:
    """Arbitrary-shape layer for edge cases (seeded like a config)."""
    W0 = normal_f32(seed + 0, (d, k), sigma_w)
    A = normal_bf16(seed + 1, (r, k), 1.0 / r)
    B = np.zeros((d, r), np.uint16) if zero_b else normal_bf16(seed + 2, (d, r), sigma_b)
    X = normal_bf16(seed + 3, (T, k), 1.0)
    dY = normal_bf16(seed + 4, (T, d), 1.0)
    return LayerInputs(W0=W0, A=A, B=B, X=X, dY=dY, d=d, k=k, r=r, T=T, s=alpha / r)


def sample_rows(seed: int, n_rows: int, count: int) -> np.ndarray:
    """Seeded sorted sample of distinct row indices (always includes the last row)."""
    gen = np.random.Generator(np.random.Philox(key=seed))
    count = min(count, n_rows)
    rows = gen.choice(n_rows, size=count, replace=False)
    rows[-1] = n_rows - 1
    return np.unique(rows)


__all__ = [
    "BASE_SEED", "TENSOR_IDS", "seed_for", "normal_f64", "normal_f32", "normal_bf16",
    "f32_to_bf16_bits", "Linear", "Config", "CONFIGS", "config", "LayerInputs",
    "make_layer", "custom_layer", "sample_rows",
]
