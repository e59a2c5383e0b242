"""tgemm_q2_noalloc: the entry point for callers that cannot allocate device memory.

Some callers may not call cudaMalloc or any allocator -- a plugin inside a host that owns
all device memory, a code path running while a stream is captured, a real-time loop.
tgemm_q2_noalloc serves them with a scratch buffer compiled into the library instead of
a caller workspace.  These tests call it through the C ABI, on two calls in a row, and
hold each result to the accuracy gates against the f64 oracle (and, as an extra check,
against tgemm_q2 with its ordinary workspace); and they check that problems too big for
the built-in buffer are refused before anything is launched.  This file is collected
last on purpose.
"""
import numpy as np
import pytest
import torch

import bit_weight_quantized_tgemm_b200 as tg
from bit_weight_quantized_tgemm_b200 import synth
from helpers import dev, gate, gate_output, out_to_f64

pytestmark = pytest.mark.gpu


def _packed(oracle, prob):
    wq, d, st = oracle.q2_pack(prob.codes, prob.scale)
    assert st == 0
    return wq, d, dev(wq, torch.uint8), dev(d, torch.float16)


def _noalloc(x, wq, d, y, out_dtype):
    return tg.lib().tgemm_q2_noalloc(x.data_ptr(), wq.data_ptr(), d.data_ptr(), y.data_ptr(),
                                     x.shape[0], wq.shape[0], x.shape[1], out_dtype,
                                     torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("M,N,K", [(300, 520, 640), (4, 256, 384)])
@pytest.mark.parametrize("out", [tg.OUT_F32, tg.OUT_BF16])
def test_noalloc_matches_oracle_twice(oracle, M, N, K, out):
    prev = tg.set_path(tg.PATH_AUTO)
    try:
        dt = torch.float32 if out == tg.OUT_F32 else torch.bfloat16
        for call in range(2):  # two calls in a row share the built-in scratch
            prob = synth.q2_problem((31, M, N, K, call), M, N, K)
            x = dev(prob.x, torch.bfloat16)
            wq_h, d_h, wq, d = _packed(oracle, prob)
            y = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
            st = _noalloc(x, wq, d, y, out)
            assert st == tg.OK, tg.lib().tgemm_strerror(st)
            y_ref = tg.gemm_q2(x, wq, d, out_dtype=out)
            torch.cuda.synchronize()
            gate_output(y, oracle.q2_gemm(prob.x, wq_h, d_h, N), oracle,
                        f"noalloc call {call} {M}x{N}x{K} against the oracle")
            gate(out_to_f64(y), out_to_f64(y_ref), f"noalloc call {call} against tgemm_q2")
    finally:
        tg.set_path(prev)


def test_noalloc_refuses_problems_beyond_its_buffer():
    # The tensor-core path needs an M*K*2-byte f16 copy of x: 4096 x 8192 x 2 = 64 MiB,
    # more than the 40 MiB buffer, so the call must return ETOOLARGE on the host.  Real
    # buffers of the stated shapes are passed, so that a regression computes in bounds
    # instead of touching memory it does not own.
    prev = tg.set_path(tg.PATH_TENSOR)
    try:
        M, N, K = 4096, 64, 8192
        x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
        wq = torch.full((N, K // 4), 0x55, dtype=torch.uint8, device="cuda")
        d = torch.zeros((N, K // 128), dtype=torch.float16, device="cuda")
        y = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
        st = _noalloc(x, wq, d, y, tg.OUT_BF16)
        torch.cuda.synchronize()
        assert st == tg.ETOOLARGE
        assert b"scratch" in tg.lib().tgemm_strerror(st)
    finally:
        tg.set_path(prev)


def test_noalloc_leaves_no_device_error():
    assert tg.device_error() == 0
