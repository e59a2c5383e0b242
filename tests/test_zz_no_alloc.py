"""tgemm_q2_noalloc: the entry point for callers that cannot allocate device memory.

Some callers may not call cudaMalloc or any allocator -- a plugin inside a host that owns
all device memory, a code path running while a stream is captured, a real-time loop.
tgemm_q2_noalloc serves them with a scratch buffer compiled into the library instead of
a caller workspace.  These tests call it through the C ABI and check that it returns what
tgemm_q2 (with its ordinary workspace) returns, within the accuracy gates the other
parity tests use, on two calls in a row; and that problems too big for the built-in
buffer are refused before anything is launched.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import bit_weight_quantized_tgemm_b200 as tg
from bit_weight_quantized_tgemm_b200 import synth
from helpers import dev, gate, out_to_f64

pytestmark = pytest.mark.gpu


def _packed(oracle, prob):
    wq, d, st = oracle.q2_pack(prob.codes, prob.scale)
    assert st == 0
    return dev(wq, torch.uint8), dev(d, torch.float16)


def _noalloc(x, wq, d, y, out_dtype):
    st = tg.lib().tgemm_q2_noalloc(x.data_ptr(), wq.data_ptr(), d.data_ptr(), y.data_ptr(),
                                   x.shape[0], wq.shape[0], x.shape[1], out_dtype,
                                   torch.cuda.current_stream().cuda_stream)
    assert st == tg.OK, tg.lib().tgemm_strerror(st)


@pytest.mark.parametrize("M,N,K", [(300, 520, 640), (4, 256, 384)])
@pytest.mark.parametrize("out", [tg.OUT_F32, tg.OUT_BF16])
def test_noalloc_matches_tgemm_q2_twice(oracle, M, N, K, out):
    prev = tg.set_path(tg.PATH_AUTO)
    try:
        dt = torch.float32 if out == tg.OUT_F32 else torch.bfloat16
        for call in range(2):  # two calls in a row share the built-in scratch
            prob = synth.q2_problem((31, M, N, K, call), M, N, K)
            x = dev(prob.x, torch.bfloat16)
            wq, d = _packed(oracle, prob)
            y_ref = tg.gemm_q2(x, wq, d, out_dtype=out)
            y = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
            _noalloc(x, wq, d, y, out)
            torch.cuda.synchronize()
            gate(out_to_f64(y), out_to_f64(y_ref), f"noalloc call {call} {M}x{N}x{K}")
    finally:
        tg.set_path(prev)


def test_noalloc_refuses_problems_beyond_its_buffer():
    # M*K*2 bytes of scratch > 40 MiB: rejected on the host, nothing launched
    P = ctypes.c_void_p
    st = tg.lib().tgemm_q2_noalloc(P(256), P(256), P(256), P(256), 4096, 64, 8192,
                                   tg.OUT_BF16, None)
    assert st == tg.ETOOLARGE
    assert b"scratch" in tg.lib().tgemm_strerror(st)


def test_noalloc_leaves_no_device_error():
    assert tg.device_error() == 0
