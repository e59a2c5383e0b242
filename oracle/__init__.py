"""CPU oracle for the ternary / 4-bit dequant-fused matmul -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline arm may
import this package.  The product path (the CUDA library and its Python binding) never
does; the two share no code.

Every function is a thin numpy wrapper around the plain C oracle in ``tgemm_oracle.c``,
which restates what the pages define:

* Q2_0 ("We're Teaching Your Browser to Paint...", section "The lucky break that wasn't
  luck"): 2-bit codes {0,1,2}, four per byte LSB first along the input axis, one f16
  scale per 128 weights, ``w = (q - 1) * d``; the scale's f32 -> f16 conversion must
  round-trip exactly.
* 4-bit format ("You Can Now Just Ask for an Image...", section "The bug that hid in one
  flipped bit"; "We're Teaching...", section "What's left"): two codes per byte, even
  index in the low nibble, ``w = (q - z) * s``.
* Side branch ("mindview-t2i-turbo", section "One step"): ``y = W x + B (A x)``.
* The matmul itself is the plain definition ``y[m,n] = sum_k w[n,k] x[m,k]`` in f64.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

PACK_BAD_CODE = 1
PACK_INEXACT = 2
PACK_NONFINITE = 4

_P = ctypes.c_void_p
_I = ctypes.c_int64

_SIGS = {
    "oracle_f16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
    "oracle_f32_to_f16_rne": (ctypes.c_uint16, [ctypes.c_float]),
    "oracle_bf16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
    "oracle_f32_to_bf16_rne": (ctypes.c_uint16, [ctypes.c_float]),
    "oracle_f64_to_bf16_rne": (ctypes.c_uint16, [ctypes.c_double]),
    "oracle_f64_to_bf16_array": (None, [_P, _I, _P]),
    "oracle_q2_unpack": (None, [_P, _I, _I, _P]),
    "oracle_q2_pack": (ctypes.c_uint32, [_P, _P, _I, _I, _P, _P]),
    "oracle_q2_from_gemlite": (ctypes.c_uint32, [_P, _P, _P, _I, _I, _I, _P, _P]),
    "oracle_q2_dequant": (None, [_P, _P, _I, _I, _P]),
    "oracle_q4_unpack": (None, [_P, _I, _I, _P]),
    "oracle_q4_pack": (ctypes.c_uint32, [_P, _P, _P, _I, _I, _P, _P]),
    "oracle_q4_dequant": (None, [_P, _P, _I, _I, _P]),
    "oracle_gemm_f64": (None, [_P, _P, _I, _I, _I, _P]),
    "oracle_lora_add_f64": (None, [_P, _P, _P, _I, _I, _I, _I, _P]),
    "oracle_q2_gemm": (None, [_P, _P, _P, _I, _I, _I, _P]),
    "oracle_q2_lora_gemm": (None, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "oracle_q4_gemm": (None, [_P, _P, _P, _I, _I, _I, _P]),
    "oracle_q2_gemm_at": (None, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _I, _P]),
    "oracle_q4_gemm_at": (None, [_P, _P, _P, _I, _I, _I, _P, _P, _I, _P]),
    "oracle_q2_dual_gemm": (None, [_P, _P, _P, _I, _P, _P, _P, _I, _I, _I, _P]),
    "oracle_q2_dual_gemm_at": (None, [_P, _P, _P, _I, _P, _P, _P, _I, _I, _I, _P, _P, _I, _P]),
    "oracle_num_threads": (ctypes.c_int, []),
}


class Oracle:
    """Handle on one build of the oracle library (the real one, or a planted mutant)."""

    def __init__(self, defines=()):
        path = _build.build(tuple(defines))
        self.path = path
        self.lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(self.lib, name)
            fn.restype = res
            fn.argtypes = args

    # ---- helpers -------------------------------------------------------------------
    @staticmethod
    def _c(a, dtype):
        a = np.ascontiguousarray(a, dtype=dtype)
        return a, a.ctypes.data_as(_P)

    # ---- scalar conversions -----------------------------------------------------------
    def f16_to_f32(self, h: int) -> float:
        return float(self.lib.oracle_f16_to_f32(int(h)))

    def f32_to_f16(self, f: float) -> int:
        return int(self.lib.oracle_f32_to_f16_rne(float(np.float32(f))))

    def bf16_to_f32(self, b: int) -> float:
        return float(self.lib.oracle_bf16_to_f32(int(b)))

    def f32_to_bf16(self, f: float) -> int:
        return int(self.lib.oracle_f32_to_bf16_rne(float(np.float32(f))))

    def f64_to_bf16(self, v) -> np.ndarray:
        v, pv = self._c(v, np.float64)
        out = np.empty(v.shape, dtype=np.uint16)
        self.lib.oracle_f64_to_bf16_array(pv, v.size, out.ctypes.data_as(_P))
        return out

    # ---- Q2_0 ------------------------------------------------------------------------
    def q2_unpack(self, wq: np.ndarray, N: int, K: int) -> np.ndarray:
        wq, p = self._c(wq, np.uint8)
        out = np.empty((N, K), dtype=np.uint8)
        self.lib.oracle_q2_unpack(p, N, K, out.ctypes.data_as(_P))
        return out

    def q2_pack(self, codes: np.ndarray, scale: np.ndarray):
        codes, pc = self._c(codes, np.uint8)
        scale, ps = self._c(scale, np.float32)
        N, K = codes.shape
        wq = np.empty((N, K // 4), dtype=np.uint8)
        d = np.empty((N, K // 128), dtype=np.uint16)
        st = self.lib.oracle_q2_pack(pc, ps, N, K, wq.ctypes.data_as(_P), d.ctypes.data_as(_P))
        return wq, d, int(st)

    def q2_from_gemlite(self, wq_g: np.ndarray, scale: np.ndarray, zero: np.ndarray, g: int):
        """gemlite-int2 (bytes [K/4][N], f32 scale and zero [N][K/g]) -> (wq, d, status)."""
        wq_g, pw = self._c(wq_g, np.uint8)
        scale, ps = self._c(scale, np.float32)
        zero, pz = self._c(zero, np.float32)
        K = wq_g.shape[0] * 4
        N = wq_g.shape[1]
        assert scale.shape == zero.shape == (N, K // g)
        assert (128 % g == 0 and g % 4 == 0) or (g % 128 == 0 and K % g == 0)
        wq = np.empty((N, K // 4), dtype=np.uint8)
        d = np.empty((N, K // 128), dtype=np.uint16)
        st = self.lib.oracle_q2_from_gemlite(pw, ps, pz, N, K, g, wq.ctypes.data_as(_P),
                                             d.ctypes.data_as(_P))
        return wq, d, int(st)

    def q2_dequant(self, wq, d, N: int, K: int) -> np.ndarray:
        wq, pw = self._c(wq, np.uint8)
        d, pd = self._c(d, np.uint16)
        out = np.empty((N, K), dtype=np.float32)
        self.lib.oracle_q2_dequant(pw, pd, N, K, out.ctypes.data_as(_P))
        return out

    # ---- 4-bit -----------------------------------------------------------------------
    def q4_unpack(self, wq: np.ndarray, N: int, K: int) -> np.ndarray:
        wq, p = self._c(wq, np.uint8)
        out = np.empty((N, K), dtype=np.uint8)
        self.lib.oracle_q4_unpack(p, N, K, out.ctypes.data_as(_P))
        return out

    def q4_pack(self, codes, s, z):
        codes, pc = self._c(codes, np.uint8)
        s, ps = self._c(s, np.float32)
        z, pz = self._c(z, np.float32)
        N, K = codes.shape
        wq = np.empty((N, K // 2), dtype=np.uint8)
        sz = np.empty((N, K // 64, 2), dtype=np.uint16)
        st = self.lib.oracle_q4_pack(pc, ps, pz, N, K, wq.ctypes.data_as(_P),
                                     sz.ctypes.data_as(_P))
        return wq, sz, int(st)

    def q4_dequant(self, wq, sz, N: int, K: int) -> np.ndarray:
        wq, pw = self._c(wq, np.uint8)
        sz, ps = self._c(sz, np.uint16)
        out = np.empty((N, K), dtype=np.float32)
        self.lib.oracle_q4_dequant(pw, ps, N, K, out.ctypes.data_as(_P))
        return out

    # ---- matmuls -----------------------------------------------------------------------
    def gemm(self, x_bf16, w_f32) -> np.ndarray:
        x, px = self._c(x_bf16, np.uint16)
        w, pw = self._c(w_f32, np.float32)
        M, K = x.shape
        N = w.shape[0]
        y = np.empty((M, N), dtype=np.float64)
        self.lib.oracle_gemm_f64(px, pw, M, N, K, y.ctypes.data_as(_P))
        return y

    def lora_add(self, x_bf16, a_bf16, b_bf16, y: np.ndarray) -> np.ndarray:
        x, px = self._c(x_bf16, np.uint16)
        a, pa = self._c(a_bf16, np.uint16)
        b, pb = self._c(b_bf16, np.uint16)
        y = np.ascontiguousarray(y, dtype=np.float64).copy()
        M, K = x.shape
        N, r = b.shape
        self.lib.oracle_lora_add_f64(px, pa, pb, r, M, N, K, y.ctypes.data_as(_P))
        return y

    def q2_gemm(self, x_bf16, wq, d, N: int) -> np.ndarray:
        x, px = self._c(x_bf16, np.uint16)
        wq, pw = self._c(wq, np.uint8)
        d, pd = self._c(d, np.uint16)
        M, K = x.shape
        y = np.empty((M, N), dtype=np.float64)
        self.lib.oracle_q2_gemm(px, pw, pd, M, N, K, y.ctypes.data_as(_P))
        return y

    def q2_lora_gemm(self, x_bf16, wq, d, a_bf16, b_bf16, N: int) -> np.ndarray:
        x, px = self._c(x_bf16, np.uint16)
        wq, pw = self._c(wq, np.uint8)
        d, pd = self._c(d, np.uint16)
        a, pa = self._c(a_bf16, np.uint16)
        b, pb = self._c(b_bf16, np.uint16)
        M, K = x.shape
        r = a.shape[0]
        y = np.empty((M, N), dtype=np.float64)
        self.lib.oracle_q2_lora_gemm(px, pw, pd, pa, pb, r, M, N, K, y.ctypes.data_as(_P))
        return y

    def q4_gemm(self, x_bf16, wq, sz, N: int) -> np.ndarray:
        x, px = self._c(x_bf16, np.uint16)
        wq, pw = self._c(wq, np.uint8)
        sz, ps = self._c(sz, np.uint16)
        M, K = x.shape
        y = np.empty((M, N), dtype=np.float64)
        self.lib.oracle_q4_gemm(px, pw, ps, M, N, K, y.ctypes.data_as(_P))
        return y

    def q2_gemm_at(self, x_bf16, wq, d, N: int, mi, ni, a_bf16=None, b_bf16=None):
        x, px = self._c(x_bf16, np.uint16)
        wq, pw = self._c(wq, np.uint8)
        d, pd = self._c(d, np.uint16)
        mi, pmi = self._c(mi, np.int64)
        ni, pni = self._c(ni, np.int64)
        M, K = x.shape
        if a_bf16 is not None:
            a, pa = self._c(a_bf16, np.uint16)
            b, pb = self._c(b_bf16, np.uint16)
            r = a.shape[0]
        else:
            pa = pb = None
            r = 0
        out = np.empty(mi.shape, dtype=np.float64)
        self.lib.oracle_q2_gemm_at(px, pw, pd, pa, pb, r, M, N, K, pmi, pni, mi.size,
                                   out.ctypes.data_as(_P))
        return out

    def q2_dual_gemm(self, x1_bf16, wq1, d1, x2_bf16, wq2, d2, N: int) -> np.ndarray:
        """y = x1 W1^T + x2 W2^T (a projection split along its input axis), f64."""
        x1, px1 = self._c(x1_bf16, np.uint16)
        wq1, pw1 = self._c(wq1, np.uint8)
        d1, pd1 = self._c(d1, np.uint16)
        x2, px2 = self._c(x2_bf16, np.uint16)
        wq2, pw2 = self._c(wq2, np.uint8)
        d2, pd2 = self._c(d2, np.uint16)
        M, K1 = x1.shape
        K2 = x2.shape[1]
        y = np.empty((M, N), dtype=np.float64)
        self.lib.oracle_q2_dual_gemm(px1, pw1, pd1, K1, px2, pw2, pd2, K2, M, N,
                                     y.ctypes.data_as(_P))
        return y

    def q2_dual_gemm_at(self, x1_bf16, wq1, d1, x2_bf16, wq2, d2, N: int, mi, ni):
        x1, px1 = self._c(x1_bf16, np.uint16)
        wq1, pw1 = self._c(wq1, np.uint8)
        d1, pd1 = self._c(d1, np.uint16)
        x2, px2 = self._c(x2_bf16, np.uint16)
        wq2, pw2 = self._c(wq2, np.uint8)
        d2, pd2 = self._c(d2, np.uint16)
        mi, pmi = self._c(mi, np.int64)
        ni, pni = self._c(ni, np.int64)
        M, K1 = x1.shape
        K2 = x2.shape[1]
        out = np.empty(mi.shape, dtype=np.float64)
        self.lib.oracle_q2_dual_gemm_at(px1, pw1, pd1, K1, px2, pw2, pd2, K2, M, N, pmi, pni,
                                        mi.size, out.ctypes.data_as(_P))
        return out

    def q4_gemm_at(self, x_bf16, wq, sz, N: int, mi, ni):
        x, px = self._c(x_bf16, np.uint16)
        wq, pw = self._c(wq, np.uint8)
        sz, ps = self._c(sz, np.uint16)
        mi, pmi = self._c(mi, np.int64)
        ni, pni = self._c(ni, np.int64)
        M, K = x.shape
        out = np.empty(mi.shape, dtype=np.float64)
        self.lib.oracle_q4_gemm_at(px, pw, ps, M, N, K, pmi, pni, mi.size,
                                   out.ctypes.data_as(_P))
        return out

    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())


_DEFAULT = None


def get() -> Oracle:
    """The real (unmutated) oracle, built on first use."""
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle()
    return _DEFAULT


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to f32 (a bit shift; no rounding involved)."""
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


__all__ = ["Oracle", "get", "bf16_bits_to_f32", "PACK_BAD_CODE", "PACK_INEXACT",
           "PACK_NONFINITE"]
