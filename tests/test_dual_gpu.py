"""Projection split along its input axis: y = x1 W1^T + x2 W2^T in one call (GPU).

The MMDiT's fused output projection reads the attention output and the MLP output
concatenated per token ("We're Teaching Your Browser to Paint", "Slice weights, not
activations"); the library computes both products into one accumulator.  Parity against
the oracle's sum of two f64 products, on both paths, ragged shapes, both schedules, and
the full MMDiT size on sampled outputs.
"""
import numpy as np
import pytest
import torch

import bit_weight_quantized_tgemm_b200 as tg
from bit_weight_quantized_tgemm_b200 import synth
from helpers import bf16_to_f32, bits16, canary_intact, dev, gate, gate_full, gate_output, nan_filled

pytestmark = pytest.mark.gpu

PATHS = {"small": tg.PATH_SMALL_M, "tensor": tg.PATH_TENSOR}


@pytest.fixture
def path():
    prev = tg.set_path(tg.PATH_AUTO)
    yield tg.set_path
    tg.set_path(prev)


def _pair(oracle, seed, M, N, K1, K2):
    p1 = synth.q2_problem((seed, 1), M, N, K1)
    p2 = synth.q2_problem((seed, 2), M, N, K2)
    wq1, d1, s1 = oracle.q2_pack(p1.codes, p1.scale)
    wq2, d2, s2 = oracle.q2_pack(p2.codes, p2.scale)
    assert s1 == 0 and s2 == 0
    host = (p1.x, wq1, d1, p2.x, wq2, d2)
    devs = (dev(p1.x, torch.bfloat16), dev(wq1, torch.uint8), dev(d1, torch.float16),
            dev(p2.x, torch.bfloat16), dev(wq2, torch.uint8), dev(d2, torch.float16))
    return host, devs


@pytest.mark.parametrize("pname", list(PATHS))
@pytest.mark.parametrize("M,N,K1,K2", [(1, 64, 128, 256), (16, 300, 256, 128), (17, 130, 128, 384),
                                       (200, 520, 640, 384), (256, 1000, 1024, 3072)])
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_dual_shapes(oracle, path, pname, M, N, K1, K2, out):
    path(PATHS[pname])
    host, devs = _pair(oracle, 31, M, N, K1, K2)
    dt = torch.float32 if out == "f32" else torch.bfloat16
    y, buf = nan_filled((M, N), dt)
    tg.gemm_q2_dual(*devs, out_dtype=tg.OUT_F32 if out == "f32" else tg.OUT_BF16, y=y)
    torch.cuda.synchronize()
    assert canary_intact(buf, M * N), "write past the end of y"
    gate_output(y, oracle.q2_dual_gemm(*host, N), oracle, f"dual {pname} {M}x{N}x({K1}+{K2}) {out}")


def test_dual_second_matrix_zero_is_single_matmul(oracle, path):
    """W2 all codes 1 (zero weights): exactly the single-input result of the same kernels."""
    path(tg.PATH_TENSOR)
    M, N, K1, K2 = 100, 256, 512, 256
    host, devs = _pair(oracle, 37, M, N, K1, K2)
    wz, dz, _ = oracle.q2_pack(np.ones((N, K2), np.uint8), np.ones((N, K2 // 128), np.float32))
    y = tg.gemm_q2_dual(devs[0], devs[1], devs[2], devs[3], dev(wz, torch.uint8),
                        dev(dz, torch.float16), out_dtype=tg.OUT_F32)
    single = tg.gemm_q2(devs[0], devs[1], devs[2], out_dtype=tg.OUT_F32)
    torch.cuda.synchronize()
    assert torch.equal(y, single)


def test_dual_split_vs_whole(oracle, path):
    """Few tiles on many SMs: split-tile and whole-tile schedules both pass, and agree."""
    path(tg.PATH_TENSOR)
    M, N, K1, K2 = 256, 512, 1024, 2048
    host, devs = _pair(oracle, 41, M, N, K1, K2)
    full = tg.dual_workspace_size(M, N, K1, K2)
    small = tg.dual_workspace_size(M, N, K1, K2, minimum=True)
    assert full > small > 0
    ref = oracle.q2_dual_gemm(*host, N)
    outs = []
    for nb in (full, small):
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        y = tg.gemm_q2_dual(*devs, out_dtype=tg.OUT_F32, workspace=ws)
        torch.cuda.synchronize()
        gate_output(y, ref, oracle, f"dual schedule ws={nb}")
        outs.append(y.cpu().numpy().astype(np.float64))
    assert np.linalg.norm(outs[0] - outs[1]) / np.linalg.norm(outs[1]) < 1e-5


@pytest.mark.slow
@pytest.mark.parametrize("M", [1536, 16])
def test_dual_mmdit_out_projection_full_size(oracle, path, M):
    """The MMDiT's fused out projection at full size: N = 3072, K1 = 3072 (attention
    output), K2 = 12288 (MLP output); bf16 out, automatic path, every output."""
    path(tg.PATH_AUTO)
    N, K1, K2 = 3072, 3072, 12288
    host, devs = _pair(oracle, 43, M, N, K1, K2)
    y = tg.gemm_q2_dual(*devs, out_dtype=tg.OUT_BF16)
    torch.cuda.synchronize()
    assert tg.device_error() == 0
    ref = oracle.q2_dual_gemm(*host, N)  # every output
    got = bf16_to_f32(bits16(y)).astype(np.float64)
    gate_full(got, bf16_to_f32(oracle.f64_to_bf16(ref)).astype(np.float64), f"dual full size M={M}")
