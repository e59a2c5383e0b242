"""The C-ABI library builds, loads and exports what include/tgemm.h declares (no GPU).

Only host-side behaviour is exercised here: symbol table, status strings, path switch,
workspace sizes and the argument checks that return before any CUDA call.
"""
import ctypes
import os
import re

import pytest

import bit_weight_quantized_tgemm_b200 as tg
from bit_weight_quantized_tgemm_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "tgemm.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    lib = tg.lib()
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), f"{n} declared in tgemm.h but not exported"


def test_binding_knows_every_symbol():
    assert set(declared_functions()) <= set(binding._SIGS)


def test_strerror_and_version():
    lib = tg.lib()
    assert lib.tgemm_strerror(0) == b"success"
    assert lib.tgemm_strerror(-5) == b"workspace missing or too small"
    assert lib.tgemm_strerror(-6).startswith(b"problem too large")
    assert lib.tgemm_strerror(-7) == b"unknown status"
    assert tg.version() >= 100


def test_set_path_roundtrip():
    prev = tg.set_path(tg.PATH_TENSOR)
    assert tg.set_path(tg.PATH_SMALL_M) == tg.PATH_TENSOR
    assert tg.set_path(prev) == tg.PATH_SMALL_M
    assert tg.lib().tgemm_set_path(7) == tg.EINVAL


def test_workspace_sizes():
    prev = tg.set_path(tg.PATH_AUTO)
    try:
        assert tg.workspace_size(tg.OP_Q2, 16, 3072, 3072) == 0          # small-M path
        assert tg.workspace_size(tg.OP_Q2, 1536, 9216, 3072) == 1536 * 3072 * 2
        lora = tg.workspace_size(tg.OP_Q2_LORA, 1536, 9216, 3072, 64)
        # f16 x + [u_hi | u_lo] + f32 partial sums of u over 6 K-slices of 512
        assert lora == 1536 * 3072 * 2 + 1536 * 128 * 2 + 6 * 1536 * 64 * 4  # wcat = 128
        # small-M path: f32 u + the partial sums
        assert tg.workspace_size(tg.OP_Q2_LORA, 4, 9216, 3072, 64) == 4 * 64 * 4  # u only
        assert tg.workspace_size(tg.OP_Q2_LORA, 1536, 9216, 3072, 0) == 0  # invalid r
        # whole tiles fill 148 SMs evenly here: minimum == full size
        assert tg.workspace_size_min(tg.OP_Q2, 1536, 9216, 3072) == 1536 * 3072 * 2
        assert tg.workspace_size_min(tg.OP_Q2_LORA, 1536, 9216, 3072, 64) == lora
        assert tg.workspace_size(9, 1, 1, 128) == 0
    finally:
        tg.set_path(prev)


def test_split_tile_workspace():
    """40 tiles of 76 stages on 148 SMs: 145 CTAs of 21 units, tiles split between them.
    The full size adds two 128 KB f32 slots per CTA and 8 counters per tile."""
    if tg.lib().tgemm_workspace_size(tg.OP_Q2, 1536, 9216, 3072, 0) == 0:
        pytest.skip("path forced elsewhere")
    x16 = 512 * 9728 * 2
    assert tg.workspace_size_min(tg.OP_Q4, 512, 2560, 9728) == x16
    if _visible_sms() not in (None, 148):
        pytest.skip("sizes below assume 148 SMs")
    slots = 2 * 145 * 128 * 256 * 4
    assert tg.workspace_size(tg.OP_Q4, 512, 2560, 9728) == x16 + slots + 40 * 8 * 4


def _visible_sms():
    import torch

    if not torch.cuda.is_available():
        return None
    return torch.cuda.get_device_properties(0).multi_processor_count


P = ctypes.c_void_p


@pytest.mark.parametrize("call", [
    lambda L: L.tgemm_q2(None, P(16), P(16), P(16), 4, 4, 128, 0, None, 0, None),
    lambda L: L.tgemm_q2(P(16), P(16), P(16), P(16), 0, 4, 128, 0, None, 0, None),
    lambda L: L.tgemm_q2(P(16), P(16), P(16), P(16), 4, 4, 100, 0, None, 0, None),
    lambda L: L.tgemm_q2(P(16), P(16), P(16), P(16), 4, 4, 128, 5, None, 0, None),
    lambda L: L.tgemm_q4(P(16), P(16), P(16), P(16), 4, 4, 96, 0, None, 0, None),
    lambda L: L.tgemm_q2_lora(P(16), P(16), P(16), P(16), P(16), 0, P(16), 4, 4, 128, 0, None, 0, None),
    lambda L: L.tgemm_q2_lora(P(16), P(16), P(16), P(16), P(16), 257, P(16), 4, 4, 128, 0, None, 0, None),
    lambda L: L.q2_pack(P(16), P(16), P(16), P(16), 4, 64, P(16), None),
    lambda L: L.q4_pack(P(16), P(16), P(16), P(16), P(16), 4, 32, P(16), None),
    lambda L: L.q2_dequant(None, P(16), P(16), 4, 128, None),
    # gemlite import: K not a multiple of 128, g neither dividing 128 nor a multiple of
    # 128 dividing K, g below 4, no rows, a missing pointer
    lambda L: L.q2_from_gemlite(P(16), P(16), P(16), 4, 96, 32, P(16), P(16), P(16), None),
    lambda L: L.q2_from_gemlite(P(16), P(16), P(16), 4, 256, 48, P(16), P(16), P(16), None),
    lambda L: L.q2_from_gemlite(P(16), P(16), P(16), 4, 256, 384, P(16), P(16), P(16), None),
    lambda L: L.q2_from_gemlite(P(16), P(16), P(16), 4, 256, 2, P(16), P(16), P(16), None),
    lambda L: L.q2_from_gemlite(P(16), P(16), P(16), 0, 256, 128, P(16), P(16), P(16), None),
    lambda L: L.q2_from_gemlite(P(16), None, P(16), 4, 256, 128, P(16), P(16), P(16), None),
    # B given transposed: no A, r out of range
    lambda L: L.tgemm_q2_lora_bt(P(16), P(16), P(16), None, P(16), 4, P(16), 4, 4, 128, 0, P(256), 1 << 20, None),
    lambda L: L.tgemm_q2_lora_bt(P(16), P(16), P(16), P(16), P(16), 0, P(16), 4, 4, 128, 0, P(256), 1 << 20, None),
    # split projection: K2 not a multiple of 128, K2 = 0, a missing second input
    lambda L: L.tgemm_q2_dual(P(16), P(16), P(16), 128, P(16), P(16), P(16), 100, P(16), 4, 4, 0, P(256), 1 << 20, None),
    lambda L: L.tgemm_q2_dual(P(16), P(16), P(16), 128, P(16), P(16), P(16), 0, P(16), 4, 4, 0, P(256), 1 << 20, None),
    lambda L: L.tgemm_q2_dual(P(16), P(16), P(16), 128, None, P(16), P(16), 128, P(16), 4, 4, 0, P(256), 1 << 20, None),
    # the dequant hooks and the no-allocation call
    lambda L: L.q4_dequant(P(16), P(16), P(16), 4, 96, None),
    lambda L: L.q2_dequant(P(16), P(16), P(16), 0, 128, None),
    lambda L: L.tgemm_q2_noalloc(P(16), P(16), P(16), P(16), 0, 4, 128, 0, None),
    lambda L: L.tgemm_q2_noalloc(P(16), P(16), None, P(16), 4, 4, 128, 0, None),
])
def test_argument_errors_return_einval(call):
    assert call(tg.lib()) == tg.EINVAL


@pytest.mark.parametrize("call", [
    lambda L: L.tgemm_q2(P(17), P(16), P(16), P(16), 4, 4, 128, 0, None, 0, None),
    lambda L: L.tgemm_q2(P(16), P(24), P(16), P(16), 4, 4, 128, 0, None, 0, None),
    lambda L: L.tgemm_q2(P(16), P(16), P(17), P(16), 4, 4, 128, 0, None, 0, None),
    lambda L: L.tgemm_q4(P(16), P(16), P(18), P(16), 4, 4, 128, 0, None, 0, None),
    lambda L: L.q2_pack(P(8), P(16), P(16), P(16), 4, 128, P(16), None),
    lambda L: L.q2_from_gemlite(P(16), P(16), P(16), 4, 256, 128, P(20), P(16), P(16), None),
    lambda L: L.q2_from_gemlite(P(16), P(18), P(16), 4, 256, 128, P(16), P(16), P(16), None),
    # the branch factors: a 4-byte, b (or bt) 2-byte aligned
    lambda L: L.tgemm_q2_lora(P(16), P(16), P(16), P(18), P(16), 4, P(16), 4, 4, 128, 0, P(256), 1 << 20, None),
    lambda L: L.tgemm_q2_lora(P(16), P(16), P(16), P(16), P(17), 4, P(16), 4, 4, 128, 0, P(256), 1 << 20, None),
    lambda L: L.tgemm_q2_lora_bt(P(16), P(16), P(16), P(16), P(17), 4, P(16), 4, 4, 128, 0, P(256), 1 << 20, None),
    # the second input of a split projection
    lambda L: L.tgemm_q2_dual(P(16), P(16), P(16), 128, P(24), P(16), P(16), 128, P(16), 4, 4, 0, P(256), 1 << 20, None),
    lambda L: L.tgemm_q2_dual(P(16), P(16), P(16), 128, P(16), P(16), P(17), 128, P(16), 4, 4, 0, P(256), 1 << 20, None),
    # a workspace that is large enough but not 256-byte aligned (tensor-core path, M = 64)
    lambda L: L.tgemm_q2(P(16), P(16), P(16), P(16), 64, 64, 128, 0, P(128), 1 << 20, None),
    # 4-bit pack: s, and the status word
    lambda L: L.q4_pack(P(16), P(18), P(16), P(16), P(16), 4, 64, P(16), None),
    lambda L: L.q4_pack(P(16), P(16), P(16), P(16), P(16), 4, 64, P(18), None),
    # the dequant hooks: wq 4-byte, w 16-byte, sz 4-byte
    lambda L: L.q2_dequant(P(18), P(16), P(16), 4, 128, None),
    lambda L: L.q2_dequant(P(16), P(16), P(24), 4, 128, None),
    lambda L: L.q4_dequant(P(16), P(18), P(16), 4, 64, None),
])
def test_misaligned_pointers_return_ealign(call):
    assert call(tg.lib()) == tg.EALIGN


def test_missing_workspace_is_reported():
    prev = tg.set_path(tg.PATH_TENSOR)
    try:
        st = tg.lib().tgemm_q2(P(256), P(256), P(256), P(256), 64, 64, 128, 0, None, 0, None)
        assert st == tg.EWORKSPACE
        st = tg.lib().tgemm_q2(P(256), P(256), P(256), P(256), 64, 64, 128, 0, P(256), 100, None)
        assert st == tg.EWORKSPACE
    finally:
        tg.set_path(prev)


def test_no_fallback_without_the_library(monkeypatch, tmp_path):
    """With libtgemm.so absent and no way to build it, the binding raises: there is no
    other implementation to fall back to."""
    from bit_weight_quantized_tgemm_b200 import build as pkg_build

    def cannot_build(*a, **k):
        raise RuntimeError("nvcc unavailable")

    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(pkg_build, "LIB", str(tmp_path / "libtgemm.so"))
    monkeypatch.setattr(pkg_build, "build", cannot_build)
    with pytest.raises(RuntimeError):
        binding.lib()
    with pytest.raises(RuntimeError):
        tg.version()


def test_noalloc_refuses_large_problems_on_the_host():
    """The no-allocation call rejects a problem whose f16 copy of x exceeds its built-in
    buffer before touching the device (2048 x 12288 x 2 bytes = 48 MiB > 40 MiB)."""
    prev = tg.set_path(tg.PATH_AUTO)
    try:
        st = tg.lib().tgemm_q2_noalloc(P(16), P(16), P(16), P(16), 2048, 64, 12288, 0, None)
        assert st == tg.ETOOLARGE
    finally:
        tg.set_path(prev)


def test_profile_read_rejects_unknown_kinds():
    import ctypes as C

    ms, n = C.c_double(), C.c_int64()
    L = tg.lib()
    assert L.tgemm_profile_read(6, C.byref(ms), C.byref(n), 0) == tg.EINVAL
    assert L.tgemm_profile_read(-1, C.byref(ms), C.byref(n), 0) == tg.EINVAL
    assert L.tgemm_profile_read(0, None, C.byref(n), 0) == tg.EINVAL


def test_dual_workspace_sizes():
    """The split projection's workspace: the f16 copies of x1 and x2 side by side per token
    ([M][K1+K2]); with 148 SMs its 144 tiles of 120 stages run whole, one per CTA, so the
    full size is the minimum.  Small M needs none."""
    L = tg.lib()
    prev = tg.set_path(tg.PATH_AUTO)
    try:
        x16 = 1536 * (3072 + 12288) * 2
        assert L.tgemm_q2_dual_workspace_size_min(1536, 3072, 3072, 12288) == x16
        assert L.tgemm_q2_dual_workspace_size(4, 3072, 3072, 12288) == 0
        assert L.tgemm_q2_dual_workspace_size_min(4, 3072, 3072, 12288) == 0
        assert L.tgemm_q2_dual_workspace_size(0, 1, 128, 128) == 0
        if _visible_sms() in (None, 148):
            # its 144 tiles of 120 stages run whole on 144 CTAs (splitting them over 148
            # would save 3 units, less than the split charge): no slots
            assert L.tgemm_q2_dual_workspace_size(1536, 3072, 3072, 12288) == x16
    finally:
        tg.set_path(prev)
