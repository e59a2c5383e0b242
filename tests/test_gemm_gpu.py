"""Matmul parity: the CUDA kernels (both paths) against the f64 CPU oracle (GPU)."""
import numpy as np
import pytest
import torch

import bit_weight_quantized_tgemm_b200 as tg
from bit_weight_quantized_tgemm_b200 import synth
from helpers import canary_intact, dev, gate, gate_output, nan_filled, out_to_f64

pytestmark = pytest.mark.gpu

PATHS = {"small": tg.PATH_SMALL_M, "tensor": tg.PATH_TENSOR}


@pytest.fixture
def path():
    prev = tg.set_path(tg.PATH_AUTO)
    yield tg.set_path
    tg.set_path(prev)


def _q2_device(prob, oracle):
    wq, d, st = oracle.q2_pack(prob.codes, prob.scale)
    assert st == 0
    return wq, d, dev(wq, torch.uint8), dev(d, torch.float16)


def _q4_device(prob, oracle):
    wq, sz, st = oracle.q4_pack(prob.codes, prob.s, prob.z)
    assert st == 0
    return wq, sz, dev(wq, torch.uint8), dev(sz, torch.float16)


def _run_q2(prob, oracle, out_dtype, lora=False):
    wq, d, twq, td = _q2_device(prob, oracle)
    x = dev(prob.x, torch.bfloat16)
    dt = torch.float32 if out_dtype == tg.OUT_F32 else torch.bfloat16
    y, buf = nan_filled((prob.M, prob.N), dt)
    if lora:
        tg.gemm_q2_lora(x, twq, td, dev(prob.a, torch.bfloat16), dev(prob.b, torch.bfloat16),
                        out_dtype=out_dtype, y=y)
        ref = oracle.q2_lora_gemm(prob.x, wq, d, prob.a, prob.b, prob.N)
    else:
        tg.gemm_q2(x, twq, td, out_dtype=out_dtype, y=y)
        ref = oracle.q2_gemm(prob.x, wq, d, prob.N)
    torch.cuda.synchronize()
    assert canary_intact(buf, prob.M * prob.N), "write past the end of y"
    return y, ref


SHAPES = [
    (1, 8, 128), (3, 40, 256), (16, 128, 256), (17, 300, 384), (100, 256, 512),
    (130, 520, 640), (256, 1000, 1024),
]


@pytest.mark.parametrize("pname", list(PATHS))
@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_q2_shapes(oracle, path, pname, M, N, K, out):
    path(PATHS[pname])
    prob = synth.q2_problem((7, M, N, K), M, N, K)
    y, ref = _run_q2(prob, oracle, tg.OUT_F32 if out == "f32" else tg.OUT_BF16)
    gate_output(y, ref, oracle, f"q2 {pname} {M}x{N}x{K} {out}")


@pytest.mark.parametrize("pname", list(PATHS))
@pytest.mark.parametrize("M,N,K", [(1, 8, 64), (5, 33, 192), (16, 64, 128), (20, 300, 320),
                                   (200, 512, 1024)])
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_q4_shapes(oracle, path, pname, M, N, K, out):
    path(PATHS[pname])
    prob = synth.q4_problem((8, M, N, K), M, N, K)
    wq, sz, twq, tsz = _q4_device(prob, oracle)
    dt = torch.float32 if out == "f32" else torch.bfloat16
    y, buf = nan_filled((M, N), dt)
    tg.gemm_q4(dev(prob.x, torch.bfloat16), twq, tsz,
               out_dtype=tg.OUT_F32 if out == "f32" else tg.OUT_BF16, y=y)
    torch.cuda.synchronize()
    assert canary_intact(buf, M * N)
    gate_output(y, oracle.q4_gemm(prob.x, wq, sz, N), oracle, f"q4 {pname} {M}x{N}x{K} {out}")


@pytest.mark.parametrize("pname", list(PATHS))
@pytest.mark.parametrize("M,N,K,r", [(4, 64, 256, 4), (16, 100, 384, 32), (40, 300, 512, 64),
                                     (130, 256, 256, 17), (64, 128, 128, 256)])
def test_q2_lora_shapes(oracle, path, pname, M, N, K, r):
    path(PATHS[pname])
    prob = synth.q2_problem((9, M, N, K, r), M, N, K, r=r, ab_sigma=0.05)
    y, ref = _run_q2(prob, oracle, tg.OUT_F32, lora=True)
    gate_output(y, ref, oracle, f"lora {pname} {M}x{N}x{K} r{r}")


@pytest.mark.parametrize("pname", list(PATHS))
def test_lora_a_only_4_byte_aligned(oracle, path, pname):
    """A at a 4-byte (not 16-byte) boundary, which the ABI allows: the branch's loads of A
    take the narrow path.  Token and K extents span several prep tiles and a ragged edge."""
    path(PATHS[pname])
    M, N, K, r = 150 if pname == "tensor" else 9, 256, 1152, 24
    prob = synth.q2_problem((22, M, N, K, r), M, N, K, r=r, ab_sigma=0.05)
    wq, d, twq, td = _q2_device(prob, oracle)
    a_dev = dev(prob.a, torch.bfloat16)
    a_buf = torch.empty(r * K + 2, dtype=torch.bfloat16, device="cuda")
    a = a_buf[2:].view(r, K)
    a.copy_(a_dev)
    assert a.data_ptr() % 16 == 4
    y, buf = nan_filled((M, N), torch.float32)
    tg.gemm_q2_lora(dev(prob.x, torch.bfloat16), twq, td, a, dev(prob.b, torch.bfloat16),
                    out_dtype=tg.OUT_F32, y=y)
    torch.cuda.synchronize()
    assert canary_intact(buf, M * N)
    gate_output(y, oracle.q2_lora_gemm(prob.x, wq, d, prob.a, prob.b, N), oracle,
                f"lora a+4B {pname}")


@pytest.mark.parametrize("pname", list(PATHS))
def test_lora_branch_alone(oracle, path, pname):
    """W == 0 (all codes 1), A, B ~ N(0,1): the output is the branch alone."""
    path(PATHS[pname])
    M, N, K, r = 48, 200, 384, 32
    prob = synth.q2_problem(21, M, N, K, r=r, ab_sigma=1.0)
    prob.codes[:] = 1
    y, ref = _run_q2(prob, oracle, tg.OUT_F32, lora=True)
    assert np.linalg.norm(ref) > 0
    gate_output(y, ref, oracle, f"lora-only {pname}")


@pytest.mark.parametrize("pname", list(PATHS))
def test_closed_forms(oracle, path, pname):
    path(PATHS[pname])
    M, N, K = 24, 96, 256
    prob = synth.q2_problem(5, M, N, K)
    prob.codes[:] = 1
    y, _ = _run_q2(prob, oracle, tg.OUT_F32)
    assert torch.all(y == 0), "all codes 1 must give exactly zero"
    prob.codes[5, 77] = 2
    prob.codes[9, 3] = 0
    y, ref = _run_q2(prob, oracle, tg.OUT_F32)
    got = out_to_f64(y)
    assert np.array_equal(got, ref), "one-hot weights are exact"


@pytest.mark.parametrize("pname", list(PATHS))
def test_q4_two_column(oracle, path, pname):
    """The pages' tiny 2-column test (golden/q4_two_column.txt) through the kernels."""
    path(PATHS[pname])
    row = [l.split() for l in open(__file__.replace("test_gemm_gpu.py", "golden/q4_two_column.txt"))
           if l.strip() and not l.startswith("#")][0]
    x0, x1, c00, c01, c10, c11, y0, y1 = (int(v) for v in row[:8])
    x = np.zeros((1, 64), np.float32)
    x[0, 0], x[0, 1] = x0, x1
    xb = dev(np.asarray(torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)), torch.bfloat16)
    codes = np.zeros((2, 64), np.uint8)
    codes[0, 0], codes[0, 1], codes[1, 0], codes[1, 1] = c00, c01, c10, c11
    one = np.ones((2, 1), np.float32)
    wq, sz, _ = oracle.q4_pack(codes, one, 0 * one)
    y = tg.gemm_q4(xb, dev(wq, torch.uint8), dev(sz, torch.float16), out_dtype=tg.OUT_F32)
    torch.cuda.synchronize()
    assert y[0].tolist() == [float(y0), float(y1)]


def test_no_device_error():
    assert tg.device_error(clear=False) == 0
