"""Small-M parity over long K (GPU): the small-M kernel covers K in passes that each fit
its shared-memory budget, and a 4-bit K may end on half a 128-weight unit.  Every output
is checked against the f64 CPU oracle, NaN-prefilled outputs and canaries included."""
import pytest
import torch

import bit_weight_quantized_tgemm_b200 as tg
from bit_weight_quantized_tgemm_b200 import synth
from helpers import canary_intact, dev, gate_output, nan_filled

pytestmark = pytest.mark.gpu


@pytest.fixture
def small_path():
    prev = tg.set_path(tg.PATH_SMALL_M)
    yield
    tg.set_path(prev)


# 16 tokens x 12288 needs four passes over K; 9 tokens takes the two-tile form; 1 token
# covers K in two passes of 6144
@pytest.mark.parametrize("M", [1, 9, 16])
@pytest.mark.parametrize("out", [tg.OUT_F32, tg.OUT_BF16])
def test_q2_long_k(oracle, small_path, M, out):
    N, K = 200, 12288
    prob = synth.q2_problem((31, M, out), M, N, K)
    wq, d, st = oracle.q2_pack(prob.codes, prob.scale)
    assert st == 0
    dt = torch.float32 if out == tg.OUT_F32 else torch.bfloat16
    y, buf = nan_filled((M, N), dt)
    tg.gemm_q2(dev(prob.x, torch.bfloat16), dev(wq, torch.uint8), dev(d, torch.float16),
               out_dtype=out, y=y)
    torch.cuda.synchronize()
    assert canary_intact(buf, M * N)
    gate_output(y, oracle.q2_gemm(prob.x, wq, d, N), oracle, f"q2 small-M {M}x{N}x{K}")


# K = 9792 is 76.5 units of 128: the last pass ends on a unit with only its first group
@pytest.mark.parametrize("M", [3, 16])
def test_q4_long_k_half_unit(oracle, small_path, M):
    N, K = 150, 9792
    prob = synth.q4_problem((32, M), M, N, K)
    wq, sz, st = oracle.q4_pack(prob.codes, prob.s, prob.z)
    assert st == 0
    y, buf = nan_filled((M, N), torch.float32)
    tg.gemm_q4(dev(prob.x, torch.bfloat16), dev(wq, torch.uint8), dev(sz, torch.float16),
               out_dtype=tg.OUT_F32, y=y)
    torch.cuda.synchronize()
    assert canary_intact(buf, M * N)
    gate_output(y, oracle.q4_gemm(prob.x, wq, sz, N), oracle, f"q4 small-M {M}x{N}x{K}")


def test_q2_lora_long_k(oracle, small_path):
    M, N, K, r = 16, 96, 12288, 8
    prob = synth.q2_problem((33, M), M, N, K, r=r, ab_sigma=0.05)
    wq, d, st = oracle.q2_pack(prob.codes, prob.scale)
    assert st == 0
    y, buf = nan_filled((M, N), torch.float32)
    tg.gemm_q2_lora(dev(prob.x, torch.bfloat16), dev(wq, torch.uint8), dev(d, torch.float16),
                    dev(prob.a, torch.bfloat16), dev(prob.b, torch.bfloat16),
                    out_dtype=tg.OUT_F32, y=y)
    torch.cuda.synchronize()
    assert canary_intact(buf, M * N)
    gate_output(y, oracle.q2_lora_gemm(prob.x, wq, d, prob.a, prob.b, N), oracle,
                f"q2 + branch small-M {M}x{N}x{K}")


# The branch operands (u of a token pass, the CTA's rows of B) sit in shared memory next to
# the activations: r = 256 at 16 tokens leaves less room for them (K is then cut into more
# passes), r = 30 and r = 1 exercise the row pitches, 33 tokens three token passes (u
# restaged per pass, the partial sums reusing the activations' space in between).
@pytest.mark.parametrize("M,N,K,r", [(1, 77, 3072, 1), (8, 130, 3072, 30), (16, 520, 3072, 256),
                                     (12, 200, 6144, 64), (33, 96, 1024, 6)])
def test_q2_lora_operands_in_shared_memory(oracle, small_path, M, N, K, r):
    prob = synth.q2_problem((34, M, N, K, r), M, N, K, r=r, ab_sigma=0.05)
    wq, d, st = oracle.q2_pack(prob.codes, prob.scale)
    assert st == 0
    args = (dev(prob.x, torch.bfloat16), dev(wq, torch.uint8), dev(d, torch.float16),
            dev(prob.a, torch.bfloat16), dev(prob.b, torch.bfloat16))
    y, buf = nan_filled((M, N), torch.float32)
    tg.gemm_q2_lora(*args, out_dtype=tg.OUT_F32, y=y)
    y2 = tg.gemm_q2_lora(*args, out_dtype=tg.OUT_F32)
    torch.cuda.synchronize()
    assert canary_intact(buf, M * N)
    gate_output(y, oracle.q2_lora_gemm(prob.x, wq, d, prob.a, prob.b, N), oracle,
                f"q2 + branch small-M {M}x{N}x{K} r{r}")
    assert torch.equal(y, y2), "two identical calls differ"
    assert tg.device_error() == 0
