"""Seeded synthetic inputs for the ternary / 4-bit matmul workloads.

This module only draws random numbers and fixes shapes.  It holds none of the method's
arithmetic (no packing, no dequantization, no matmul), so the CUDA path and the CPU
oracle can both be fed from it without sharing any computation.

Draw order inside one problem (numpy ``default_rng``): activations X, codes, scales,
zeros, low-rank A, low-rank B.  Activations are drawn in f32 and rounded to bf16 by
torch (round to nearest, ties to even); scales and zeros are drawn in f32 and rounded to
f16 by numpy, so every scale handed to the packers is exactly representable in f16 (the
converter's exact-roundtrip rule in "We're Teaching Your Browser to Paint...", section
"The lucky break that wasn't luck").  ``N(0, s)`` means standard deviation ``s``.

Workloads (sizes and distributions of the pages' linears):

* ``tiny``      -- 16 x 256 activations, 128 x 256 ternary weights, f32 output.
* ``gemv``      -- M in {1, 4, 16} tokens through one 3072 x 3072 ternary matrix,
                   codes P(0)=P(2)=0.3, P(1)=0.4 (the HBM-bound small-M case).
* ``mmdit``     -- 1536 tokens (1024 image + 512 text) through the MMDiT's ternary
                   shapes 9216x3072, 3072x12288 and 12288x3072 (N x K).
* ``lora``      -- the 9216 x 3072 shape plus a rank-r side branch, r in {4, 32, 64},
                   A and B ~ N(0, 1e-3).
* ``encoder``   -- 512 tokens through the 4-bit encoder linears 9728x2560 (up) and
                   2560x9728 (down), group 64, s = |N(0, 0.01)|, z ~ U[7, 8].
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np


def _bf16_bits(a: np.ndarray) -> np.ndarray:
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def _f16_exact(a: np.ndarray) -> np.ndarray:
    return np.asarray(a, dtype=np.float32).astype(np.float16).astype(np.float32)


@dataclass
class Q2Problem:
    x: np.ndarray            # bf16 bits [M, K]
    codes: np.ndarray        # uint8 [N, K], values in {0, 1, 2}
    scale: np.ndarray        # f32 [N, K/128], each exactly an f16 value
    a: Optional[np.ndarray] = None  # bf16 bits [r, K]
    b: Optional[np.ndarray] = None  # bf16 bits [N, r]
    out_f32: bool = False
    seed: object = None

    @property
    def M(self):
        return self.x.shape[0]

    @property
    def N(self):
        return self.codes.shape[0]

    @property
    def K(self):
        return self.codes.shape[1]

    @property
    def r(self):
        return 0 if self.a is None else self.a.shape[0]


@dataclass
class Q4Problem:
    x: np.ndarray            # bf16 bits [M, K]
    codes: np.ndarray        # uint8 [N, K], values 0..15
    s: np.ndarray            # f32 [N, K/64], exactly f16
    z: np.ndarray            # f32 [N, K/64], exactly f16
    out_f32: bool = False
    seed: object = None

    @property
    def M(self):
        return self.x.shape[0]

    @property
    def N(self):
        return self.codes.shape[0]

    @property
    def K(self):
        return self.codes.shape[1]


def q2_problem(seed, M: int, N: int, K: int, *, code_probs=None, d_sigma: float = 0.02,
               x_sigma: float = 1.0, r: int = 0, ab_sigma: float = 1e-3,
               out_f32: bool = False) -> Q2Problem:
    """One seeded ternary problem.  ``code_probs`` = (P0, P1, P2) or None for uniform."""
    if K % 128:
        raise ValueError("K must be a multiple of 128 for Q2_0")
    rng = np.random.default_rng(seed)
    x = _bf16_bits(rng.standard_normal((M, K), dtype=np.float32) * np.float32(x_sigma))
    if code_probs is None:
        codes = rng.integers(0, 3, size=(N, K), dtype=np.uint8)
    else:
        codes = rng.choice(3, size=(N, K), p=list(code_probs)).astype(np.uint8)
    scale = _f16_exact(np.abs(rng.standard_normal((N, K // 128), dtype=np.float32)
                              * np.float32(d_sigma)))
    a = b = None
    if r:
        a = _bf16_bits(rng.standard_normal((r, K), dtype=np.float32) * np.float32(ab_sigma))
        b = _bf16_bits(rng.standard_normal((N, r), dtype=np.float32) * np.float32(ab_sigma))
    return Q2Problem(x=x, codes=codes, scale=scale, a=a, b=b, out_f32=out_f32, seed=seed)


def q4_problem(seed, M: int, N: int, K: int, *, s_sigma: float = 0.01, z_lo: float = 7.0,
               z_hi: float = 8.0, x_sigma: float = 1.0, out_f32: bool = False) -> Q4Problem:
    if K % 64:
        raise ValueError("K must be a multiple of 64 for the 4-bit format")
    rng = np.random.default_rng(seed)
    x = _bf16_bits(rng.standard_normal((M, K), dtype=np.float32) * np.float32(x_sigma))
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    s = _f16_exact(np.abs(rng.standard_normal((N, K // 64), dtype=np.float32)
                          * np.float32(s_sigma)))
    z = _f16_exact(rng.uniform(z_lo, z_hi, size=(N, K // 64)).astype(np.float32))
    return Q4Problem(x=x, codes=codes, s=s, z=z, out_f32=out_f32, seed=seed)


# ---- the named workloads ------------------------------------------------------------

@dataclass
class Workload:
    name: str
    kind: str                 # "q2", "q2_lora" or "q4"
    M: int
    N: int
    K: int
    seed: object
    r: int = 0
    out_f32: bool = False
    code_probs: Optional[tuple] = None
    extra: dict = field(default_factory=dict)

    def make(self):
        if self.kind == "q4":
            return q4_problem(self.seed, self.M, self.N, self.K, out_f32=self.out_f32)
        return q2_problem(self.seed, self.M, self.N, self.K, code_probs=self.code_probs,
                          r=self.r, out_f32=self.out_f32)

    @property
    def flops(self) -> int:
        f = 2 * self.M * self.N * self.K
        if self.r:
            f += 2 * self.M * self.r * (self.K + self.N)
        return f

    @property
    def weight_bytes(self) -> int:
        """Packed-weight bytes: codes plus scales (2.125 or 4.5 bits per weight)."""
        if self.kind == "q4":
            return self.N * self.K // 2 + self.N * (self.K // 64) * 4
        return self.N * self.K // 4 + self.N * (self.K // 128) * 2


# Seeds: one per workload family (0 tiny, 1 GEMV, 2 MMDiT, 3 branch, 4 encoder); every shape
# of a family draws its own problem from a fresh generator with the family's seed.
TINY = [Workload("tiny", "q2", 16, 128, 256, seed=0, out_f32=True)]
GEMV = [Workload(f"gemv_m{m}", "q2", m, 3072, 3072, seed=1,
                 code_probs=(0.3, 0.4, 0.3)) for m in (1, 4, 16)]
MMDIT = [Workload(f"mmdit_{n}x{k}", "q2", 1536, n, k, seed=2)
         for n, k in ((9216, 3072), (3072, 12288), (12288, 3072))]
LORA = [Workload(f"lora_r{r}", "q2_lora", 1536, 9216, 3072, seed=3, r=r) for r in (4, 32, 64)]
ENCODER = [Workload("encoder_up", "q4", 512, 9728, 2560, seed=4),
           Workload("encoder_down", "q4", 512, 2560, 9728, seed=4)]

ALL = {w.name: w for w in TINY + GEMV + MMDIT + LORA + ENCODER}
