"""Failure detection on the GPU without a fault: a wait that nothing satisfies must give
up after the library's wait limit, report TGEMM_DEVERR_TIMEOUT through the device error
word, and leave the context usable for the next matmul (GPU)."""
import time

import pytest
import torch

import bit_weight_quantized_tgemm_b200 as tg
from bit_weight_quantized_tgemm_b200 import synth
from helpers import dev, gate_output

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(oracle):
    tg.device_error(clear=True)
    t0 = time.monotonic()
    tg.selftest_wait_timeout()
    bits = tg.device_error(clear=True)  # synchronizes the device
    waited = time.monotonic() - t0
    assert bits & tg.DEVERR_TIMEOUT, f"device error word {bits:#x}: the wait did not report"
    assert waited >= 0.5, f"the wait gave up after {waited:.3f} s, before its limit"
    assert waited < 30.0
    assert tg.device_error() == 0, "the error word did not clear"

    # the context is intact: a matmul on each path still matches the oracle
    prob = synth.q2_problem(41, 130, 260, 384)
    wq, d, st = oracle.q2_pack(prob.codes, prob.scale)
    assert st == 0
    for path in (tg.PATH_SMALL_M, tg.PATH_TENSOR):
        prev = tg.set_path(path)
        try:
            y = tg.gemm_q2(dev(prob.x, torch.bfloat16), dev(wq, torch.uint8), dev(d, torch.float16),
                           out_dtype=tg.OUT_F32)
            torch.cuda.synchronize()
        finally:
            tg.set_path(prev)
        gate_output(y, oracle.q2_gemm(prob.x, wq, d, prob.N), oracle, f"after the timeout, path {path}")
    assert tg.device_error() == 0


def test_launch_errors_are_reported_by_the_call_that_made_them(oracle):
    """A launch the runtime refuses on the host returns TGEMM_ECUDA from that call; the
    error it leaves behind in the runtime's last-error slot is not charged to the next,
    valid call, which returns TGEMM_OK and computes correctly."""
    st = tg.lib().tgemm_selftest_bad_launch(torch.cuda.current_stream().cuda_stream)
    assert st == tg.ECUDA
    prob = synth.q2_problem(43, 40, 136, 256)
    wq, d, _ = oracle.q2_pack(prob.codes, prob.scale)
    prev = tg.set_path(tg.PATH_AUTO)
    try:
        # raises on any status other than TGEMM_OK
        y = tg.gemm_q2(dev(prob.x, torch.bfloat16), dev(wq, torch.uint8), dev(d, torch.float16),
                       out_dtype=tg.OUT_F32)
        torch.cuda.synchronize()
    finally:
        tg.set_path(prev)
    gate_output(y, oracle.q2_gemm(prob.x, wq, d, prob.N), oracle, "after a refused launch")
    assert tg.device_error() == 0
