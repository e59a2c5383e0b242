"""The low-rank branch with B given transposed (bt [r][N], the model file's ".bt") (GPU).

On both paths, tgemm_q2_lora_bt must give bit for bit the result of tgemm_q2_lora on the
transposed copy. It must also pass the accuracy gates against the oracle, which reads B
as bt transposed. Ragged N and r cover the element-by-element load path; r a multiple
of 8 with B rows 16-byte aligned covers the vector path of the B layout.
"""
import numpy as np
import pytest
import torch

import bit_weight_quantized_tgemm_b200 as tg
from bit_weight_quantized_tgemm_b200 import synth
from helpers import dev, gate_output

pytestmark = pytest.mark.gpu

PATHS = {"small": tg.PATH_SMALL_M, "tensor": tg.PATH_TENSOR}


@pytest.fixture
def path():
    prev = tg.set_path(tg.PATH_AUTO)
    yield tg.set_path
    tg.set_path(prev)


@pytest.mark.parametrize("pname", list(PATHS))
@pytest.mark.parametrize("M,N,K,r", [(1, 64, 128, 1), (5, 300, 256, 4), (16, 130, 384, 17),
                                     (200, 520, 640, 64), (300, 1000, 1152, 32), (129, 257, 512, 8)])
def test_bt_equals_b_layout(oracle, path, pname, M, N, K, r):
    path(PATHS[pname])
    prob = synth.q2_problem((81, M, N, K, r), M, N, K, r=r)
    wq, d, st = oracle.q2_pack(prob.codes, prob.scale)
    assert st == 0
    x, twq, td = dev(prob.x, torch.bfloat16), dev(wq, torch.uint8), dev(d, torch.float16)
    a = dev(prob.a, torch.bfloat16)
    bt_host = np.ascontiguousarray(prob.b.T)                         # [r][N]
    b = dev(prob.b, torch.bfloat16)                                  # [N][r]
    bt = dev(bt_host, torch.bfloat16)
    y_b = tg.gemm_q2_lora(x, twq, td, a, b, out_dtype=tg.OUT_F32)
    y_bt = tg.gemm_q2_lora_bt(x, twq, td, a, bt, out_dtype=tg.OUT_F32)
    torch.cuda.synchronize()
    assert tg.device_error() == 0
    assert torch.equal(y_b, y_bt), "B^T input differs from the B input"
    # the oracle reads B [N][r]: the transpose of bt, taken here by numpy
    ref = oracle.q2_lora_gemm(prob.x, wq, d, prob.a, np.ascontiguousarray(bt_host.T), N)
    gate_output(y_bt, ref, oracle, f"branch with B^T, {pname} {M}x{N}x{K} r={r}")


def test_bt_shape_is_checked():
    x = torch.zeros(4, 128, dtype=torch.bfloat16, device="cuda")
    wq = torch.zeros(64, 32, dtype=torch.uint8, device="cuda")
    d = torch.zeros(64, 1, dtype=torch.float16, device="cuda")
    a = torch.zeros(4, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        tg.gemm_q2_lora_bt(x, wq, d, a, torch.zeros(64, 4, dtype=torch.bfloat16, device="cuda"))
