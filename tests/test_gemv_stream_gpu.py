"""The small-M streaming kernel on the GPU: parity with the oracle over the shapes that
select each of its launch plans, and the orderings it relies on (GPU).

Shapes are chosen so that the plans cover one and several passes over K (partial sums
kept across passes), ring depths below and at 4, ragged row counts (N not a multiple of 8
or 32), a CTA holding several 32-row tiles, the 4-bit K that ends on half a unit, 1 to 16
tokens and both output types.  Outputs are pre-filled with NaN and followed by
canary words.  Further checks:
- a call whose activations are the previous call's output on the same stream (the kernel
  reads x only after its dependency wait, while its weight copies start before it);
- device packing followed at once by the matmul, no synchronization between them (the
  packers let no later kernel start before they finish);
- the per-pass kernel gives the same result within the gates (an independent check of the
  new kernel's k order and correction sums);
- a burst of back-to-back calls over alternating weights, checked at the end.
"""
import numpy as np
import pytest
import torch

import bit_weight_quantized_tgemm_b200 as tg
from bit_weight_quantized_tgemm_b200 import synth
from helpers import canary_intact, dev, gate, gate_output, nan_filled, out_to_f64

pytestmark = pytest.mark.gpu

CASES = [
    # fmt, M, N, K
    (0, 1, 136, 256), (0, 16, 136, 256), (0, 5, 1000, 640), (0, 9, 3072, 3072),
    (0, 16, 520, 12288), (0, 3, 1, 128), (0, 8, 2000, 1024), (0, 12, 77, 384),
    (1, 5, 1000, 576), (1, 16, 1000, 576), (1, 13, 520, 12288), (1, 2, 7, 64),
    (1, 1, 4100, 2560), (1, 16, 2560, 9728), (0, 2, 21504, 3072), (0, 16, 520, 65536),
]


@pytest.fixture(autouse=True)
def stream_path():
    # the streaming form wherever its layout fits (the automatic choice takes it only for
    # the shapes where it measured faster)
    prev = tg.set_path(tg.PATH_SMALL_M_STREAM)
    yield
    tg.set_path(prev)


def _problem(oracle, fmt, M, N, K, seed):
    if fmt == 0:
        prob = synth.q2_problem((61, seed, M, N, K), M, N, K, code_probs=(0.3, 0.4, 0.3))
        wq, sc, st = oracle.q2_pack(prob.codes, prob.scale)
        ref = lambda xb: oracle.q2_gemm(xb, wq, sc, N)  # noqa: E731
        return prob, dev(wq, torch.uint8), dev(sc, torch.float16), ref
    prob = synth.q4_problem((62, seed, M, N, K), M, N, K)
    wq, sc, st = oracle.q4_pack(prob.codes, prob.s, prob.z)
    ref = lambda xb: oracle.q4_gemm(xb, wq, sc, N)  # noqa: E731
    return prob, dev(wq, torch.uint8), dev(sc, torch.float16), ref


def _call(fmt, x, wq, sc, out_dtype, y=None):
    if fmt == 0:
        return tg.gemm_q2(x, wq, sc, out_dtype=out_dtype, y=y)
    return tg.gemm_q4(x, wq, sc, out_dtype=out_dtype, y=y)


def test_cases_cover_the_plans():
    plans = [tg.gemv_plan(f, M, N, K) for f, M, N, K in CASES]
    assert all(p is not None for p in plans)
    passes = {p["passes"] for p in plans}
    assert 1 in passes and len(passes - {1}) >= 2, passes
    assert {p["T"] for p in plans} == {1, 2}
    assert min(p["S"] for p in plans) < 4 and max(p["S"] for p in plans) == 4


@pytest.mark.parametrize("fmt,M,N,K", CASES)
@pytest.mark.parametrize("out", [tg.OUT_F32, tg.OUT_BF16])
def test_stream_matches_oracle(oracle, fmt, M, N, K, out):
    prob, wq, sc, ref = _problem(oracle, fmt, M, N, K, 0)
    dt = torch.float32 if out == tg.OUT_F32 else torch.bfloat16
    y, buf = nan_filled((M, N), dt)
    _call(fmt, dev(prob.x, torch.bfloat16), wq, sc, out, y)
    torch.cuda.synchronize()
    assert canary_intact(buf, M * N), "the kernel wrote past y"
    gate_output(y, ref(prob.x), oracle, f"stream fmt={fmt} {M}x{N}x{K}")
    assert tg.device_error() == 0


@pytest.mark.parametrize("fmt,M,N,K", [(0, 16, 3072, 3072), (1, 7, 1000, 576), (0, 4, 520, 12288)])
def test_stream_agrees_with_pass_kernel(oracle, fmt, M, N, K):
    prob, wq, sc, _ = _problem(oracle, fmt, M, N, K, 1)
    x = dev(prob.x, torch.bfloat16)
    y_new = _call(fmt, x, wq, sc, tg.OUT_F32)
    tg.set_path(tg.PATH_SMALL_M_PASS)
    y_old = _call(fmt, x, wq, sc, tg.OUT_F32)
    torch.cuda.synchronize()
    gate(out_to_f64(y_new), out_to_f64(y_old), f"stream vs pass fmt={fmt}")


def test_chained_call_reads_the_previous_output(oracle):
    """y1 = x0 W1^T, then y2 = y1 W2^T on the same stream without a sync: the second call's
    activations are the first call's output."""
    M, K = 6, 1024
    p1, w1, d1, _ = _problem(oracle, 0, M, K, K, 2)
    p2 = synth.q2_problem((63, 2), 1, 2048, K)
    w2h, d2h, _ = oracle.q2_pack(p2.codes, p2.scale)
    x0 = dev(p1.x, torch.bfloat16)
    y1 = tg.gemm_q2(x0, w1, d1, out_dtype=tg.OUT_BF16)
    y2 = tg.gemm_q2(y1, dev(w2h, torch.uint8), dev(d2h, torch.float16), out_dtype=tg.OUT_F32)
    torch.cuda.synchronize()
    y1_bits = y1.cpu().view(torch.int16).numpy().view(np.uint16)
    gate_output(y2, oracle.q2_gemm(y1_bits, w2h, d2h, 2048), oracle, "second call of a chain")


@pytest.mark.parametrize("fmt", [0, 1])
def test_pack_then_matmul_without_sync(oracle, fmt):
    M, N, K = 9, 1000, 1024
    if fmt == 0:
        prob = synth.q2_problem((64, 0), M, N, K)
        wq_h, sc_h, _ = oracle.q2_pack(prob.codes, prob.scale)
        wq, sc, st = tg.q2_pack(torch.from_numpy(prob.codes).cuda(), torch.from_numpy(prob.scale).cuda())
        y = tg.gemm_q2(dev(prob.x, torch.bfloat16), wq, sc, out_dtype=tg.OUT_F32)
        ref = oracle.q2_gemm(prob.x, wq_h, sc_h, N)
    else:
        prob = synth.q4_problem((64, 1), M, N, K)
        wq_h, sc_h, _ = oracle.q4_pack(prob.codes, prob.s, prob.z)
        wq, sc, st = tg.q4_pack(torch.from_numpy(prob.codes).cuda(), torch.from_numpy(prob.s).cuda(),
                                torch.from_numpy(prob.z).cuda())
        y = tg.gemm_q4(dev(prob.x, torch.bfloat16), wq, sc, out_dtype=tg.OUT_F32)
        ref = oracle.q4_gemm(prob.x, wq_h, sc_h, N)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    gate_output(y, ref, oracle, f"pack then matmul fmt={fmt}")


def test_burst_of_calls(oracle):
    """40 back-to-back calls alternating two weight matrices and two inputs; the last two
    outputs are checked."""
    M, N, K = 16, 3072, 3072
    pa, wa, da, refa = _problem(oracle, 0, M, N, K, 3)
    pb, wb, db, refb = _problem(oracle, 0, M, N, K, 4)
    xa, xb = dev(pa.x, torch.bfloat16), dev(pb.x, torch.bfloat16)
    ya = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    yb = torch.empty_like(ya)
    for i in range(20):
        tg.gemm_q2(xa, wa, da, out_dtype=tg.OUT_BF16, y=ya)
        tg.gemm_q2(xb, wb, db, out_dtype=tg.OUT_BF16, y=yb)
    torch.cuda.synchronize()
    gate_output(ya, refa(pa.x), oracle, "burst, first matrix")
    gate_output(yb, refb(pb.x), oracle, "burst, second matrix")
    assert tg.device_error() == 0
