"""Seeded synthetic activation workloads.

Both the CPU oracle (through the tests) and the CUDA path consume the arrays made here;
this module holds none of the quantizer's arithmetic (no rotation, no scale rule, no
rounding to FP4).  It only draws random numbers and casts fp32 to bf16 bit patterns.

The workloads stand in for "activations of LLM linear layers", which the pages evaluate
on real models (Llama-3, Qwen-3) that are not available here.  Their shapes follow the
hidden sizes of such layers (4096, 8192, 14336).

Recipe (fixed order, one ``numpy.random.default_rng(seed)`` per workload):
  1. outlier-channel indices: ``rng.choice(K, n_outlier, replace=False)``;
  2. per-row factors (only the log-normal workload): ``rng.lognormal(0, sigma, M)``;
  3. the body, drawn row-chunk by row-chunk in row-major order (the stream is the same
     as drawing the whole matrix at once);
  4. the outlier columns are multiplied by their factor;
  5. fp32 -> bf16 with round-to-nearest-even on the bit pattern.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Iterator, Optional

import numpy as np

MXFP4 = 0
NVFP4 = 1

SCALE_FLOOR_OCP = 0
SCALE_CEIL_NOCLIP = 1
SCALE_OAS = 2
SCALE_NV_STATIC = 3
SCALE_NV_DYNAMIC = 4

RULE_NAMES = {
    SCALE_FLOOR_OCP: "floor",
    SCALE_CEIL_NOCLIP: "ceil",
    SCALE_OAS: "oas",
    SCALE_NV_STATIC: "nv_static",
    SCALE_NV_DYNAMIC: "nv_dynamic",
}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round-to-nearest, ties to even) and return the
    16-bit patterns as uint16.  Inputs are finite and far from the bf16 overflow edge."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    # finite inputs keep u + 0x8000 below 2**32, so uint32 arithmetic does not wrap
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic activation matrix X (M x K, bf16) and the quantizer setting it is
    measured with."""

    name: str
    M: int
    K: int
    seed: int
    body: str  # "normal" | "student_t"
    n_outlier: int
    outlier_scale: float
    row_lognormal_sigma: float = 0.0
    student_t_nu: float = 3.0
    body_scale: float = 1.0
    fmt: int = MXFP4
    group: int = 32
    block: int = 32
    rule: int = SCALE_FLOOR_OCP

    @property
    def numel(self) -> int:
        return self.M * self.K

    def with_quantizer(self, fmt: int, group: int, block: int, rule: int, name: Optional[str] = None) -> "Workload":
        return dataclasses.replace(self, fmt=fmt, group=group, block=block, rule=rule, name=name or self.name)

    def with_rows(self, M: int, name: Optional[str] = None) -> "Workload":
        return dataclasses.replace(self, M=M, name=name or self.name)

    def row_chunks(self, chunk_rows: int = 1024) -> Iterator[np.ndarray]:
        """Yield X as consecutive row chunks of bf16 bit patterns (uint16, row-major)."""
        rng = np.random.default_rng(self.seed)
        K = self.K
        outl = rng.choice(K, self.n_outlier, replace=False) if self.n_outlier else np.zeros(0, np.int64)
        row_fac = None
        if self.row_lognormal_sigma > 0.0:
            row_fac = rng.lognormal(0.0, self.row_lognormal_sigma, self.M).astype(np.float32)
        col_fac = np.ones(K, np.float32)
        col_fac[outl] = np.float32(self.outlier_scale)
        for r0 in range(0, self.M, chunk_rows):
            r1 = min(self.M, r0 + chunk_rows)
            n = r1 - r0
            if self.body == "normal":
                body = rng.standard_normal((n, K), dtype=np.float32)
            elif self.body == "student_t":
                body = rng.standard_t(self.student_t_nu, (n, K)).astype(np.float32)
            else:
                raise ValueError(self.body)
            if self.body_scale != 1.0:
                body *= np.float32(self.body_scale)
            if row_fac is not None:
                body *= row_fac[r0:r1, None]
            body *= col_fac[None, :]
            yield f32_to_bf16_bits(body)

    def generate(self) -> np.ndarray:
        """X as one (M, K) uint16 array of bf16 bit patterns."""
        out = np.empty((self.M, self.K), np.uint16)
        r = 0
        for ch in self.row_chunks():
            out[r:r + ch.shape[0]] = ch
            r += ch.shape[0]
        return out

    def outlier_columns(self) -> np.ndarray:
        rng = np.random.default_rng(self.seed)
        return rng.choice(self.K, self.n_outlier, replace=False) if self.n_outlier else np.zeros(0, np.int64)

    def bytes_per_call(self) -> int:
        """Algorithmic bytes of one rotate+quantize call: bf16 input, packed codes, scales
        (plus the 4-byte fp32 tensor scale for NVFP4)."""
        n = self.numel
        b = 2 * n + n // 2 + n // self.group
        if self.fmt == NVFP4:
            b += 4
        return b


def _outliers(frac: float, K: int) -> int:
    return int(round(frac * K))


# The five workloads.  Names give format, group, block, rule and shape.
SMALL_MX = Workload("mxfp4_g32_b32_floor_128x4096", 128, 4096, 0, "normal", 8, 50.0,
                    fmt=MXFP4, group=32, block=32, rule=SCALE_FLOOR_OCP)
NV_4K = Workload("nvfp4_g16_b16_4096x4096", 4096, 4096, 1, "normal", _outliers(0.005, 4096), 50.0,
                 fmt=NVFP4, group=16, block=16, rule=SCALE_NV_STATIC)
MX_8K_FLOOR = Workload("mxfp4_g32_b128_floor_8192x8192_t3", 8192, 8192, 2, "student_t", 0, 1.0,
                       student_t_nu=3.0, body_scale=0.5, fmt=MXFP4, group=32, block=128, rule=SCALE_FLOOR_OCP)
MX_8K_CEIL = MX_8K_FLOOR.with_quantizer(MXFP4, 32, 128, SCALE_CEIL_NOCLIP, "mxfp4_g32_b128_ceil_8192x8192_t3")
DECODE = tuple(
    Workload(f"mxfp4_g32_b32_floor_decode_{m}x14336", m, 14336, 3, "normal", 16, 100.0,
             fmt=MXFP4, group=32, block=32, rule=SCALE_FLOOR_OCP)
    for m in (1, 4, 16))
PREFILL_NV = Workload("nvfp4_g16_b128_prefill_32768x14336", 32768, 14336, 4, "normal", _outliers(0.005, 14336), 50.0,
                      row_lognormal_sigma=1.0, fmt=NVFP4, group=16, block=128, rule=SCALE_NV_STATIC)
PREFILL_MX = PREFILL_NV.with_quantizer(MXFP4, 32, 128, SCALE_FLOOR_OCP, "mxfp4_g32_b128_floor_prefill_32768x14336")

ALL = (SMALL_MX, NV_4K, MX_8K_FLOOR, MX_8K_CEIL) + DECODE + (PREFILL_NV, PREFILL_MX)
BY_NAME = {w.name: w for w in ALL}


def lcm(a: int, b: int) -> int:
    return a * b // math.gcd(a, b)


def random_sign_mask(K: int, seed: int) -> np.ndarray:
    """Random per-channel sign bits for a randomised Hadamard rotation: ceil(K / 32) uint32
    words from ``numpy.random.default_rng(seed)``, bits at or above K cleared.  (Bit k of
    word k // 32 set means channel k is negated; the library and the oracle each read the
    bits themselves.)"""
    n = (K + 31) // 32
    w = np.random.default_rng(seed).integers(0, 1 << 32, size=n, dtype=np.uint64).astype(np.uint32)
    if K % 32:
        w[-1] &= np.uint32((1 << (K % 32)) - 1)
    return w


def synthetic_weights(N: int, K: int, seed: int) -> np.ndarray:
    """Synthetic weight matrix W (N x K bf16 bit patterns): Laplace(0, 0.02) entries, the
    heavy-tailed shape the error analysis assigns to LLM weights, with 0.5 % of the input
    channels scaled by 10 (outlier channels)."""
    rng = np.random.default_rng(seed)
    cols = rng.choice(K, max(1, round(0.005 * K)), replace=False)
    w = rng.laplace(0.0, 0.02, size=(N, K)).astype(np.float32)
    w[:, cols] *= np.float32(10.0)
    return f32_to_bf16_bits(w)
