"""Seeded synthetic inputs for exact attention, shared by the CUDA path and the oracle.

This module draws random numbers and rounds them to 16-bit storage formats. It
holds none of the attention arithmetic: no scores, no softmax, no products. Both
the GPU tests and the fp64 oracle receive exactly the same 16-bit values, the
oracle as their exact float32 widening.

Recipe (the pages run their examples on no dataset; these stand in for "sequences
of thousands to tens of thousands of tokens, multi-head"):

* numpy ``default_rng(seed)`` (PCG64), ``standard_normal(dtype=float32)``;
* draw order Q, K, V, dO, each of shape [B, H, N, d];
* optional large-logit rows: per (b, h), ``floor(frac * N)`` distinct query rows
  chosen with the same generator (``rng.choice(N, size, replace=False)``) are
  multiplied by ``factor`` (a power of two, so it commutes with the rounding);
* float32 -> bf16 or fp16 by round-to-nearest-even.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

GENERATOR_VERSION = 1

BF16 = "bf16"
FP16 = "fp16"


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round-to-nearest-even (finite inputs)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) >> 16
    return u.astype(np.uint16)


def round_to_fp16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> IEEE binary16 bit patterns (numpy's conversion is round-to-nearest-even)."""
    return np.ascontiguousarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


def widen(bits: np.ndarray, dtype: str) -> np.ndarray:
    """16-bit patterns -> their exact float32 values."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    if dtype == BF16:
        return (bits.astype(np.uint32) << 16).view(np.float32)
    if dtype == FP16:
        return bits.view(np.float16).astype(np.float32)
    raise ValueError(f"unknown dtype {dtype!r}")


def to_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == BF16:
        return round_to_bf16_bits(x)
    if dtype == FP16:
        return round_to_fp16_bits(x)
    raise ValueError(f"unknown dtype {dtype!r}")


@dataclass
class AttnInputs:
    """Raw 16-bit inputs, each uint16 of shape [B, H, N, d]."""

    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    do: np.ndarray
    dtype: str
    seed: int
    large_rows: np.ndarray | None = None  # [B*H, n_large] row indices scaled up, or None

    @property
    def shape(self):
        return self.q.shape

    def widened(self, name: str) -> np.ndarray:
        return widen(getattr(self, name), self.dtype)


def make_inputs(B: int, H: int, N: int, d: int, dtype: str = BF16, seed: int = 0,
                large_frac: float = 0.0, large_factor: float = 8.0,
                with_do: bool = True) -> AttnInputs:
    """Draw Q, K, V (and dO) iid N(0, 1) from ``seed`` and round them to ``dtype``."""
    rng = np.random.default_rng(seed)
    shape = (B, H, N, d)
    q = rng.standard_normal(shape, dtype=np.float32)
    k = rng.standard_normal(shape, dtype=np.float32)
    v = rng.standard_normal(shape, dtype=np.float32)
    do = rng.standard_normal(shape, dtype=np.float32) if with_do else np.zeros(shape, np.float32)
    large = None
    if large_frac > 0.0:
        n_large = int(math.floor(large_frac * N))
        large = np.empty((B * H, n_large), dtype=np.int64)
        qf = q.reshape(B * H, N, d)
        for bh in range(B * H):
            rows = rng.choice(N, size=n_large, replace=False)
            large[bh] = rows
            qf[bh, rows, :] *= np.float32(large_factor)
    return AttnInputs(q=to_bits(q, dtype), k=to_bits(k, dtype), v=to_bits(v, dtype),
                      do=to_bits(do, dtype), dtype=dtype, seed=seed, large_rows=large)


# The five workloads named for this method. Seeds are 1000 * config id (+ sweep index).
@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str
    causal: bool
    seed: int
    large_frac: float = 0.0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def fwd_flops(self) -> float:
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def make(self, with_do: bool = True) -> AttnInputs:
        return make_inputs(self.B, self.H, self.N, self.d, self.dtype, self.seed,
                           self.large_frac, 8.0, with_do)


def config_seed(config_id: int, sweep_index: int = 0) -> int:
    return 1000 * config_id + sweep_index


WORKLOADS = {
    "c1": Workload("c1 B1 H1 N256 d64 bf16 non-causal", 1, 1, 256, 64, BF16, False, config_seed(1)),
    "c2": Workload("c2 B4 H16 N2048 d64 bf16 non-causal", 4, 16, 2048, 64, BF16, False, config_seed(2)),
    "c2c": Workload("c2 B4 H16 N2048 d64 bf16 causal", 4, 16, 2048, 64, BF16, True, config_seed(2)),
    "c3": Workload("c3 B2 H32 N8192 d128 bf16 causal", 2, 32, 8192, 128, BF16, True, config_seed(3)),
    "c4": Workload("c4 B1 H16 N65536 d128 bf16 causal, 1% rows x8", 1, 16, 65536, 128, BF16, True,
                   config_seed(4), large_frac=0.01),
    # c3 with a sequence length that is not a multiple of 128 (the last tile of every
    # head is partial): the ragged-N path at the headline size
    "c3r": Workload("c3r B2 H32 N8000 d128 bf16 causal", 2, 32, 8000, 128, BF16, True,
                    config_seed(3, 1)),
}


def sweep_workloads():
    """Config 5: N in {512..16384}, B*N = 16384 tokens, H=16, d in {64,128}, fp16/bf16, causal/non."""
    out = []
    idx = 0
    for N in (512, 1024, 2048, 4096, 8192, 16384):
        for d in (64, 128):
            for dtype in (BF16, FP16):
                for causal in (False, True):
                    out.append(Workload(f"c5 N{N} d{d} {dtype} {'causal' if causal else 'non-causal'}",
                                        16384 // N, 16, N, d, dtype, causal, config_seed(5, idx)))
                    idx += 1
    return out
