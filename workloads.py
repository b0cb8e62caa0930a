"""Seeded synthetic inputs for the BitLinear W1.58A8 forward.

This module only draws random numbers and lays them out; it performs none of
the method's arithmetic (no absmean, no absmax, no rounding to codes).  It is
the one module that both the CPU oracle side and the CUDA side read, so that
the two are fed the same arrays.

Recipe (shapes and distributions follow the five workload descriptions of the
BitLinear W1.58A8 decode/prefill study):

* Full-precision latent weights ``W`` are ``0.02 * N(0, 1)`` in fp32, shape
  ``[N, K]`` (nn.Linear layout: row ``n`` is output feature ``n``).
* Activations ``x`` are ``N(0, 1)`` in fp32, shape ``[M, K]``.  Where a
  workload asks for outlier channels, ``floor(0.01 * K)`` channels picked by a
  seeded permutation are multiplied by 20 (every token, same channels).
* Where a workload asks for bf16 activations the fp32 values are rounded to
  bf16 (round to nearest, ties to even) and both sides receive the same bf16
  bit patterns.

Every generator is ``numpy.random.Generator(PCG64(seed))``.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

WEIGHT_STD = 0.02
OUTLIER_FRACTION = 0.01
OUTLIER_SCALE = 20.0


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def latent_weights(seed: int, n: int, k: int, std: float = WEIGHT_STD) -> np.ndarray:
    """fp32 ``[n, k]`` drawn as ``std * N(0, 1)`` (scaled in fp32)."""
    w = _rng(seed).standard_normal((n, k), dtype=np.float32)
    w *= np.float32(std)
    return w


def activations(seed: int, m: int, k: int, outliers: bool = False) -> np.ndarray:
    """fp32 ``[m, k]`` drawn as ``N(0, 1)``; optional 1% outlier channels x20."""
    g = _rng(seed)
    x = g.standard_normal((m, k), dtype=np.float32)
    if outliers:
        n_out = int(np.floor(OUTLIER_FRACTION * k))
        ch = g.permutation(k)[:n_out]
        x[:, ch] *= np.float32(OUTLIER_SCALE)
    return x


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns the uint16 bit patterns.

    Input preparation only (the workload says the activations *are* bf16);
    inputs here are finite, so NaN handling is not needed.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 exactly."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


@dataclass(frozen=True)
class Shape:
    """One BitLinear call: ``y[M, N] = BitLinear(x[M, K])`` with weights ``[N, K]``."""
    name: str
    M: int
    K: int
    N: int
    w_seed: int
    x_seed: int
    x_dtype: str = "f32"       # "f32" or "bf16"
    y_dtype: str = "f32"       # "f32" or "bf16"
    outliers: bool = False

    def weights(self) -> np.ndarray:
        return latent_weights(self.w_seed, self.N, self.K)

    def inputs(self) -> np.ndarray:
        """fp32 activations; for bf16 workloads these are the widened bf16 values."""
        x = activations(self.x_seed, self.M, self.K, self.outliers)
        if self.x_dtype == "bf16":
            return bf16_to_f32(bf16_bits(x))
        return x

    def inputs_bf16_bits(self) -> np.ndarray:
        assert self.x_dtype == "bf16"
        return bf16_bits(activations(self.x_seed, self.M, self.K, self.outliers))

    @property
    def packed_bytes(self) -> int:
        return self.N * (self.K // 16) * 4

    @property
    def algorithmic_bytes(self) -> int:
        """Packed weights read + activations read + output written."""
        xb = 2 if self.x_dtype == "bf16" else 4
        yb = 2 if self.y_dtype == "bf16" else 4
        return self.packed_bytes + self.M * self.K * xb + self.M * self.N * yb

    @property
    def ops(self) -> int:
        """2 ops per multiply-accumulate, counted densely over all N*K weights."""
        return 2 * self.M * self.N * self.K


@dataclass(frozen=True)
class Workload:
    name: str
    description: str
    shapes: tuple = field(default_factory=tuple)


# Workload 1: single BitLinear, M=1, K=N=1024, fp32 in/out.
W1 = Workload("m1_k1024_n1024", "single BitLinear forward, M=1, K=1024, N=1024, fp32 x and y",
              (Shape("m1_k1024_n1024", 1, 1024, 1024, 1001, 2001),))

# Workload 2: decode GEMV, M=1, bf16 activations with 1% outlier channels, the
# FFN up (K=4096 -> N=11008) and down (K=11008 -> N=4096) shapes.
W2 = Workload("decode_m1_ffn_up_down_bf16",
              "decode GEMV M=1, bf16 x with 1% x20 outlier channels; K=4096,N=11008 and K=11008,N=4096",
              (Shape("up_k4096_n11008", 1, 4096, 11008, 1002, 2002, "bf16", "f32", True),
               Shape("down_k11008_n4096", 1, 11008, 4096, 1012, 2012, "bf16", "f32", True)))

# Workload 3: small-batch decode, M in {4, 16, 64}, K=4096, N in {4096, 11008}.
W3 = Workload("decode_small_batch", "M in {4,16,64}, K=4096, N in {4096,11008}, fp32 x and y",
              tuple(Shape(f"m{m}_k4096_n{n}", m, 4096, n, 1003 + 10 * i, 2003 + 10 * i)
                    for i, (m, n) in enumerate([(m, n) for m in (4, 16, 64) for n in (4096, 11008)])))

# Workload 4: prefill GEMM, M=2048, K=4096, N in {4096, 11008}, bf16 output,
# activations with outlier channels quantised per token.
W4 = Workload("prefill_m2048", "prefill GEMM M=2048, K=4096, N in {4096,11008}; int8 per-token x; bf16 y",
              (Shape("prefill_k4096_n4096", 2048, 4096, 4096, 1004, 2004, "f32", "bf16", True),
               Shape("prefill_k4096_n11008", 2048, 4096, 11008, 1014, 2014, "f32", "bf16", True)))

# Workload 5: one decoder block at batch-1 decode, hidden 2560, intermediate 6912.
BLOCK_HIDDEN = 2560
BLOCK_INTER = 6912
BLOCK_PROJ = ("q", "k", "v", "o", "gate", "up", "down")


def block_shapes() -> dict:
    """Weight shapes ``(N, K)`` and seeds of the seven block projections."""
    h, f = BLOCK_HIDDEN, BLOCK_INTER
    nk = {"q": (h, h), "k": (h, h), "v": (h, h), "o": (h, h),
          "gate": (f, h), "up": (f, h), "down": (h, f)}
    return {p: (nk[p][0], nk[p][1], 1050 + i) for i, p in enumerate(BLOCK_PROJ)}


def block_weights() -> dict:
    return {p: latent_weights(seed, n, k) for p, (n, k, seed) in block_shapes().items()}


def block_input() -> np.ndarray:
    return activations(2005, 1, BLOCK_HIDDEN)


WORKLOADS = {w.name: w for w in (W1, W2, W3, W4)}
