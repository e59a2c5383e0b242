"""Thin ctypes binding over libtgemm.so (include/tgemm.h).

Argument marshalling only: every function checks tensor dtype/device/contiguity, passes
``data_ptr()`` values and the current CUDA stream to the C entry point of the same name,
and raises :class:`TgemmError` on a nonzero status.  All computation happens in the CUDA
kernels.  There is no fallback: if the shared library is missing or fails to load,
every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

from . import build as _build

OK, EINVAL, EALIGN, ECUDA, EARCH, EWORKSPACE, ETOOLARGE = 0, -1, -2, -3, -4, -5, -6
NOALLOC_SCRATCH_BYTES = 40 * 1024 * 1024
OUT_F32, OUT_BF16 = 0, 1
OP_Q2, OP_Q2_LORA, OP_Q4 = 0, 1, 2
PATH_AUTO, PATH_SMALL_M, PATH_TENSOR, PATH_SMALL_M_PASS, PATH_SMALL_M_STREAM = 0, 1, 2, 3, 4
PACK_BAD_CODE, PACK_INEXACT, PACK_NONFINITE = 1, 2, 4
PACK_ZERO_MISMATCH, PACK_GROUP_MISMATCH = 8, 16
DEVERR_TIMEOUT = 1
KIND_TC_Q2, KIND_TC_Q2_LORA, KIND_TC_Q4, KIND_GEMV_Q2, KIND_GEMV_Q4, KIND_PREP = range(6)

_P = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t

_SIGS = {
    "q2_pack": (_i, [_P, _P, _P, _P, _i, _i, _P, _P]),
    "q4_pack": (_i, [_P, _P, _P, _P, _P, _i, _i, _P, _P]),
    "q2_from_gemlite": (_i, [_P, _P, _P, _i, _i, _i, _P, _P, _P, _P]),
    "q2_dequant": (_i, [_P, _P, _P, _i, _i, _P]),
    "q4_dequant": (_i, [_P, _P, _P, _i, _i, _P]),
    "tgemm_selftest_wait_timeout": (_i, [_P]),
    "tgemm_selftest_bad_launch": (_i, [_P]),
    "tgemm_gemv_plan": (_i, [_i, _i, _i, _i, _i, _P]),
    "tgemm_mma_rate": (_i, [_i, _i, _i, _P, _i, _P]),
    "tgemm_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "tgemm_workspace_size_min": (_sz, [_i, _i, _i, _i, _i]),
    "tgemm_q2_dual_workspace_size": (_sz, [_i, _i, _i, _i]),
    "tgemm_q2_dual_workspace_size_min": (_sz, [_i, _i, _i, _i]),
    "tgemm_tc_plan": (_i, [_i, _i, _i, _i, _i, _i, _i, _P]),
    "tgemm_q2": (_i, [_P, _P, _P, _P, _i, _i, _i, _i, _P, _sz, _P]),
    "tgemm_q2_lora": (_i, [_P, _P, _P, _P, _P, _i, _P, _i, _i, _i, _i, _P, _sz, _P]),
    "tgemm_q2_lora_bt": (_i, [_P, _P, _P, _P, _P, _i, _P, _i, _i, _i, _i, _P, _sz, _P]),
    "tgemm_q4": (_i, [_P, _P, _P, _P, _i, _i, _i, _i, _P, _sz, _P]),
    "tgemm_q2_dual": (_i, [_P, _P, _P, _i, _P, _P, _P, _i, _P, _i, _i, _i, _P, _sz, _P]),
    "tgemm_q2_noalloc": (_i, [_P, _P, _P, _P, _i, _i, _i, _i, _P]),
    "tgemm_strerror": (ctypes.c_char_p, [_i]),
    "tgemm_set_path": (_i, [_i]),
    "tgemm_device_error": (_i, [_P, _i]),
    "tgemm_version": (_i, []),
    "tgemm_profile_enable": (_i, [_i]),
    "tgemm_profile_read": (_i, [_i, _P, _P, _i]),
    "tgemm_launch_count": (ctypes.c_int64, []),
}


class TgemmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        try:
            msg = lib().tgemm_strerror(status).decode()
        except Exception:  # pragma: no cover - only if the library itself is unusable
            msg = "?"
        super().__init__(f"{where}: status {status} ({msg})")


_lib = None
_lock = threading.Lock()


def library_path() -> str:
    return _build.LIB


def lib():
    """Load libtgemm.so (building it first if the sources are newer)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                path = _build.LIB
                if not os.path.exists(path) or _build.stale():
                    _build.build()
                handle = ctypes.CDLL(path)
                for name, (res, args) in _SIGS.items():
                    fn = getattr(handle, name)
                    fn.restype = res
                    fn.argtypes = args
                _lib = handle
    return _lib


def _check(status: int, where: str):
    if status != OK:
        raise TgemmError(status, where)


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, dtype, name: str):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


# ---- packing ----------------------------------------------------------------------------

def q2_pack(codes: torch.Tensor, scale: torch.Tensor, status: Optional[torch.Tensor] = None):
    """codes uint8 [N, K], scale f32 [N, K/128] -> (wq uint8 [N, K/4], d f16 [N, K/128], status)."""
    _need(codes, torch.uint8, "codes")
    _need(scale, torch.float32, "scale")
    N, K = codes.shape
    wq = torch.empty((N, K // 4), dtype=torch.uint8, device=codes.device)
    d = torch.empty((N, K // 128), dtype=torch.float16, device=codes.device)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=codes.device)
    _check(lib().q2_pack(_ptr(codes), _ptr(scale), _ptr(wq), _ptr(d), N, K, _ptr(status),
                         _stream()), "q2_pack")
    return wq, d, status


def q2_from_gemlite(wq_g: torch.Tensor, scale: torch.Tensor, zero: torch.Tensor, g: int,
                    status: Optional[torch.Tensor] = None):
    """gemlite-int2 bytes uint8 [K/4, N], f32 scale and zero [N, K/g] -> Q2_0
    (wq uint8 [N, K/4], d f16 [N, K/128], status); see q2_from_gemlite in tgemm.h."""
    _need(wq_g, torch.uint8, "wq_g")
    _need(scale, torch.float32, "scale")
    _need(zero, torch.float32, "zero")
    K4, N = wq_g.shape
    K = 4 * K4
    if g < 1 or K % g or tuple(scale.shape) != (N, K // g) or tuple(zero.shape) != (N, K // g):
        raise ValueError("scale and zero must be [N, K/g]")
    wq = torch.empty((N, K4), dtype=torch.uint8, device=wq_g.device)
    d = torch.empty((N, K // 128), dtype=torch.float16, device=wq_g.device)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=wq_g.device)
    _check(lib().q2_from_gemlite(_ptr(wq_g), _ptr(scale), _ptr(zero), N, K, g, _ptr(wq), _ptr(d),
                                 _ptr(status), _stream()), "q2_from_gemlite")
    return wq, d, status


def q4_pack(codes: torch.Tensor, s: torch.Tensor, z: torch.Tensor,
            status: Optional[torch.Tensor] = None):
    """codes uint8 [N, K], s, z f32 [N, K/64] -> (wq uint8 [N, K/2], sz f16 [N, K/64, 2], status)."""
    _need(codes, torch.uint8, "codes")
    _need(s, torch.float32, "s")
    _need(z, torch.float32, "z")
    N, K = codes.shape
    wq = torch.empty((N, K // 2), dtype=torch.uint8, device=codes.device)
    sz = torch.empty((N, K // 64, 2), dtype=torch.float16, device=codes.device)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=codes.device)
    _check(lib().q4_pack(_ptr(codes), _ptr(s), _ptr(z), _ptr(wq), _ptr(sz), N, K, _ptr(status),
                         _stream()), "q4_pack")
    return wq, sz, status


def q2_dequant(wq: torch.Tensor, d: torch.Tensor) -> torch.Tensor:
    _need(wq, torch.uint8, "wq")
    _need(d, torch.float16, "d")
    N, K = wq.shape[0], wq.shape[1] * 4
    w = torch.empty((N, K), dtype=torch.float32, device=wq.device)
    _check(lib().q2_dequant(_ptr(wq), _ptr(d), _ptr(w), N, K, _stream()), "q2_dequant")
    return w


def q4_dequant(wq: torch.Tensor, sz: torch.Tensor) -> torch.Tensor:
    _need(wq, torch.uint8, "wq")
    _need(sz, torch.float16, "sz")
    N, K = wq.shape[0], wq.shape[1] * 2
    w = torch.empty((N, K), dtype=torch.float32, device=wq.device)
    _check(lib().q4_dequant(_ptr(wq), _ptr(sz), _ptr(w), N, K, _stream()), "q4_dequant")
    return w


# ---- matmuls --------------------------------------------------------------------------------

def selftest_wait_timeout() -> None:
    """Launch the failure-detection self test on the current stream: a wait that can never
    be satisfied gives up after the library's wait limit (1 s) and sets DEVERR_TIMEOUT."""
    _check(lib().tgemm_selftest_wait_timeout(_stream()), "tgemm_selftest_wait_timeout")


def workspace_size(op: int, M: int, N: int, K: int, r: int = 0) -> int:
    return int(lib().tgemm_workspace_size(op, M, N, K, r))


def workspace_size_min(op: int, M: int, N: int, K: int, r: int = 0) -> int:
    """Smallest accepted workspace (whole tiles per CTA); see tgemm_workspace_size_min."""
    return int(lib().tgemm_workspace_size_min(op, M, N, K, r))


TC_PLAN_KEYS = ("tiles_m", "num_tiles", "ksteps", "sk_t0", "upc", "dpc", "grid", "split")


def tc_plan(op: int, M: int, N: int, K: int, r: int = 0, K2: int = 0, sms: int = 148) -> dict:
    """The tensor-core kernel's schedule for these sizes on `sms` SMs (tgemm_tc_plan)."""
    out = (ctypes.c_int * len(TC_PLAN_KEYS))()
    _check(lib().tgemm_tc_plan(op, M, N, K, r, K2, sms, out), "tgemm_tc_plan")
    return dict(zip(TC_PLAN_KEYS, out))


GEMV_PLAN_KEYS = ("T", "kp", "passes", "grid", "S", "U", "j_max", "smem", "nbox", "xs_stride",
                  "off_x", "off_corr", "off_red", "off_acc", "off_sc", "off_ring", "off_bar")


def gemv_plan(fmt: int, M: int, N: int, K: int, sms: int = 148):
    """The small-M streaming kernel's launch plan (tgemm_gemv_plan), or None when no
    layout fits and the per-pass kernel serves the call."""
    out = (ctypes.c_int * len(GEMV_PLAN_KEYS))()
    st = lib().tgemm_gemv_plan(fmt, M, N, K, sms, out)
    if st == ETOOLARGE:
        return None
    _check(st, "tgemm_gemv_plan")
    return dict(zip(GEMV_PLAN_KEYS, out))


def mma_rate(mode: int, n: int = 16, iters: int = 4096) -> float:
    """Cycles per operation of tgemm_mma_rate's `mode` (averaged over the SMs)."""
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    out = torch.zeros(sms, dtype=torch.int64, device="cuda")
    _check(lib().tgemm_mma_rate(mode, n, iters, _ptr(out), sms, _stream()), "tgemm_mma_rate")
    torch.cuda.synchronize()
    return float(out.double().mean().item()) / iters


_ws_cache = {}


def _workspace(op, M, N, K, r, device, workspace):
    need = workspace_size(op, M, N, K, r)
    if need == 0:
        return None, 0
    if workspace is not None:
        _need(workspace, torch.uint8, "workspace")
        return workspace, workspace.numel()
    key = (device.index if device.index is not None else torch.cuda.current_device())
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < need:
        buf = torch.empty(need, dtype=torch.uint8, device=device)
        _ws_cache[key] = buf
    return buf, buf.numel()


def _out(y, M, N, out_dtype, device):
    dt = torch.float32 if out_dtype == OUT_F32 else torch.bfloat16
    if y is None:
        return torch.empty((M, N), dtype=dt, device=device)
    _need(y, dt, "y")
    if tuple(y.shape) != (M, N):
        raise ValueError(f"y must have shape {(M, N)}")
    return y


def gemm_q2(x: torch.Tensor, wq: torch.Tensor, d: torch.Tensor, *, out_dtype: int = OUT_BF16,
            y: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None):
    """y = x . W^T, x bf16 [M, K], W packed Q2_0 (wq uint8 [N, K/4], d f16 [N, K/128])."""
    _need(x, torch.bfloat16, "x")
    _need(wq, torch.uint8, "wq")
    _need(d, torch.float16, "d")
    M, K = x.shape
    N = wq.shape[0]
    y = _out(y, M, N, out_dtype, x.device)
    ws, nbytes = _workspace(OP_Q2, M, N, K, 0, x.device, workspace)
    _check(lib().tgemm_q2(_ptr(x), _ptr(wq), _ptr(d), _ptr(y), M, N, K, out_dtype, _ptr(ws),
                          nbytes, _stream()), "tgemm_q2")
    return y


def gemm_q2_noalloc(x: torch.Tensor, wq: torch.Tensor, d: torch.Tensor, *,
                    out_dtype: int = OUT_BF16, y: Optional[torch.Tensor] = None):
    """gemm_q2 through tgemm_q2_noalloc: scratch comes from the library's built-in buffer.

    For callers that cannot allocate device memory (pass a preallocated ``y``).  Calls
    that overlap on the GPU share that buffer and race; see include/tgemm.h."""
    _need(x, torch.bfloat16, "x")
    _need(wq, torch.uint8, "wq")
    _need(d, torch.float16, "d")
    M, K = x.shape
    N = wq.shape[0]
    y = _out(y, M, N, out_dtype, x.device)
    _check(lib().tgemm_q2_noalloc(_ptr(x), _ptr(wq), _ptr(d), _ptr(y), M, N, K, out_dtype,
                                  _stream()), "tgemm_q2_noalloc")
    return y


def gemm_q2_lora(x, wq, d, a, b, *, out_dtype: int = OUT_BF16, y=None, workspace=None):
    """y = x . W^T + (x . A^T) . B^T with a bf16 [r, K], b bf16 [N, r]."""
    _need(x, torch.bfloat16, "x")
    _need(wq, torch.uint8, "wq")
    _need(d, torch.float16, "d")
    _need(a, torch.bfloat16, "a")
    _need(b, torch.bfloat16, "b")
    M, K = x.shape
    N = wq.shape[0]
    r = a.shape[0]
    if tuple(a.shape) != (r, K) or tuple(b.shape) != (N, r):
        raise ValueError(f"a must be [r, K] and b [N, r]; got {tuple(a.shape)}, {tuple(b.shape)}")
    y = _out(y, M, N, out_dtype, x.device)
    ws, nbytes = _workspace(OP_Q2_LORA, M, N, K, r, x.device, workspace)
    _check(lib().tgemm_q2_lora(_ptr(x), _ptr(wq), _ptr(d), _ptr(a), _ptr(b), r, _ptr(y), M, N,
                               K, out_dtype, _ptr(ws), nbytes, _stream()), "tgemm_q2_lora")
    return y


def gemm_q2_lora_bt(x, wq, d, a, bt, *, out_dtype: int = OUT_BF16, y=None, workspace=None):
    """gemm_q2_lora with B given transposed: bt bf16 [r, N] (see tgemm_q2_lora_bt)."""
    _need(x, torch.bfloat16, "x")
    _need(wq, torch.uint8, "wq")
    _need(d, torch.float16, "d")
    _need(a, torch.bfloat16, "a")
    _need(bt, torch.bfloat16, "bt")
    M, K = x.shape
    N = wq.shape[0]
    r = a.shape[0]
    if tuple(a.shape) != (r, K) or tuple(bt.shape) != (r, N):
        raise ValueError(f"a must be [r, K] and bt [r, N]; got {tuple(a.shape)}, {tuple(bt.shape)}")
    y = _out(y, M, N, out_dtype, x.device)
    ws, nbytes = _workspace(OP_Q2_LORA, M, N, K, r, x.device, workspace)
    _check(lib().tgemm_q2_lora_bt(_ptr(x), _ptr(wq), _ptr(d), _ptr(a), _ptr(bt), r, _ptr(y), M,
                                  N, K, out_dtype, _ptr(ws), nbytes, _stream()), "tgemm_q2_lora_bt")
    return y


def dual_workspace_size(M: int, N: int, K1: int, K2: int, minimum: bool = False) -> int:
    """Workspace bytes for gemm_q2_dual (fastest schedule, or the accepted minimum)."""
    fn = lib().tgemm_q2_dual_workspace_size_min if minimum else lib().tgemm_q2_dual_workspace_size
    return int(fn(M, N, K1, K2))


def gemm_q2_dual(x1, wq1, d1, x2, wq2, d2, *, out_dtype: int = OUT_BF16, y=None, workspace=None):
    """y = x1 . W1^T + x2 . W2^T: a projection split along its input axis, one kernel."""
    for t, dt, nm in ((x1, torch.bfloat16, "x1"), (wq1, torch.uint8, "wq1"), (d1, torch.float16, "d1"),
                      (x2, torch.bfloat16, "x2"), (wq2, torch.uint8, "wq2"), (d2, torch.float16, "d2")):
        _need(t, dt, nm)
    M, K1 = x1.shape
    K2 = x2.shape[1]
    N = wq1.shape[0]
    if x2.shape[0] != M or wq2.shape[0] != N:
        raise ValueError("x1/x2 must have the same tokens and W1/W2 the same rows")
    y = _out(y, M, N, out_dtype, x1.device)
    need = dual_workspace_size(M, N, K1, K2)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x1.device)
    if workspace is not None:
        _need(workspace, torch.uint8, "workspace")
    nbytes = workspace.numel() if workspace is not None else 0
    _check(lib().tgemm_q2_dual(_ptr(x1), _ptr(wq1), _ptr(d1), K1, _ptr(x2), _ptr(wq2), _ptr(d2),
                               K2, _ptr(y), M, N, out_dtype, _ptr(workspace), nbytes, _stream()),
           "tgemm_q2_dual")
    return y


def gemm_q4(x, wq, sz, *, out_dtype: int = OUT_BF16, y=None, workspace=None):
    """y = x . W^T for 4-bit weights (wq uint8 [N, K/2], sz f16 [N, K/64, 2])."""
    _need(x, torch.bfloat16, "x")
    _need(wq, torch.uint8, "wq")
    _need(sz, torch.float16, "sz")
    M, K = x.shape
    N = wq.shape[0]
    y = _out(y, M, N, out_dtype, x.device)
    ws, nbytes = _workspace(OP_Q4, M, N, K, 0, x.device, workspace)
    _check(lib().tgemm_q4(_ptr(x), _ptr(wq), _ptr(sz), _ptr(y), M, N, K, out_dtype, _ptr(ws),
                          nbytes, _stream()), "tgemm_q4")
    return y


# ---- control -------------------------------------------------------------------------------

def set_path(path: int) -> int:
    prev = lib().tgemm_set_path(path)
    if prev < 0:
        raise TgemmError(prev, "tgemm_set_path")
    return prev


def device_error(clear: bool = False) -> int:
    bits = ctypes.c_uint32(0)
    _check(lib().tgemm_device_error(ctypes.addressof(bits), 1 if clear else 0),
           "tgemm_device_error")
    return int(bits.value)


def version() -> int:
    return int(lib().tgemm_version())


PROFILE_ALL = (1 << 6) - 1


def profile_enable(kinds) -> int:
    """Record CUDA events around launches of the kernel kinds in the bit mask ``kinds``
    (``True`` = every kind, ``False`` = none; see tgemm_profile_enable).  Returns the
    previous mask."""
    if kinds is True:
        kinds = PROFILE_ALL
    elif kinds is False or kinds is None:
        kinds = 0
    return int(lib().tgemm_profile_enable(int(kinds)))


def profile_read(kind: int, reset: bool = True):
    """(total device ms, launches) recorded for kernel kind `kind` (KIND_*)."""
    ms = ctypes.c_double(0.0)
    n = ctypes.c_int64(0)
    _check(lib().tgemm_profile_read(kind, ctypes.addressof(ms), ctypes.addressof(n),
                                    1 if reset else 0), "tgemm_profile_read")
    return float(ms.value), int(n.value)


def launch_count() -> int:
    """Kernels launched by libtgemm.so since it was loaded."""
    return int(lib().tgemm_launch_count())
