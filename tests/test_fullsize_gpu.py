"""Full-size parity: every matmul of the benchmark step at its benchmark size (GPU).

Each workload runs exactly as bench.py launches it:
- the automatic path choice;
- the full workspace from tgemm_workspace_size, so the split-tile schedule is used where
  it is chosen;
- bf16 output;
- weights packed on the device.

The device pack must equal the oracle's pack byte for byte. Then EVERY output is compared
with the oracle's whole-matrix result (f64, rounded to bf16) under the accuracy gates; a
failure names the worst 256-token x 32-row blocks (one TMEM lane quarter of a tensor-core
tile), so a striped fault cannot hide in a sample.
"""
import numpy as np
import pytest
import torch

import bit_weight_quantized_tgemm_b200 as tg
from bit_weight_quantized_tgemm_b200 import synth
from helpers import bf16_to_f32, bits16, dev, gate, gate_full

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

STEP = ["mmdit_9216x3072", "mmdit_3072x12288", "mmdit_12288x3072", "lora_r4", "lora_r32",
        "lora_r64", "encoder_up", "encoder_down", "gemv_m1", "gemv_m4", "gemv_m16"]


@pytest.fixture(autouse=True)
def auto_path():
    prev = tg.set_path(tg.PATH_AUTO)
    yield
    tg.set_path(prev)


def _packed_q2(oracle, prob):
    wq_o, d_o, st = oracle.q2_pack(prob.codes, prob.scale)
    assert st == 0
    twq, td, tst = tg.q2_pack(torch.from_numpy(prob.codes).cuda(), torch.from_numpy(prob.scale).cuda())
    torch.cuda.synchronize()
    assert int(tst.item()) == 0
    assert np.array_equal(twq.cpu().numpy(), wq_o), "device Q2 pack differs from the oracle"
    assert np.array_equal(bits16(td), d_o), "device scale pack differs from the oracle"
    return wq_o, d_o, twq, td


@pytest.mark.parametrize("name", STEP)
def test_step_matmul_full_size(oracle, name):
    w = synth.ALL[name]
    prob = w.make()
    M, N, K = w.M, w.N, w.K
    x = dev(prob.x, torch.bfloat16)
    if w.kind == "q4":
        wq_o, sz_o, st = oracle.q4_pack(prob.codes, prob.s, prob.z)
        assert st == 0
        twq, tsz, tst = tg.q4_pack(torch.from_numpy(prob.codes).cuda(), torch.from_numpy(prob.s).cuda(),
                                   torch.from_numpy(prob.z).cuda())
        torch.cuda.synchronize()
        assert int(tst.item()) == 0
        assert np.array_equal(twq.cpu().numpy(), wq_o), "device 4-bit pack differs from the oracle"
        assert np.array_equal(bits16(tsz), sz_o), "device (s, z) pack differs from the oracle"
        ws = torch.empty(max(tg.workspace_size(tg.OP_Q4, M, N, K), 256), dtype=torch.uint8, device="cuda")
        y = tg.gemm_q4(x, twq, tsz, out_dtype=tg.OUT_BF16, workspace=ws)
        torch.cuda.synchronize()
        ref = oracle.q4_gemm(prob.x, wq_o, sz_o, N)
    else:
        wq_o, d_o, twq, td = _packed_q2(oracle, prob)
        if w.kind == "q2_lora":
            op, r = tg.OP_Q2_LORA, w.r
        else:
            op, r = tg.OP_Q2, 0
        ws = torch.empty(max(tg.workspace_size(op, M, N, K, r), 256), dtype=torch.uint8, device="cuda")
        if r:
            y = tg.gemm_q2_lora(x, twq, td, dev(prob.a, torch.bfloat16), dev(prob.b, torch.bfloat16),
                                out_dtype=tg.OUT_BF16, workspace=ws)
            torch.cuda.synchronize()
            ref = oracle.q2_lora_gemm(prob.x, wq_o, d_o, prob.a, prob.b, N)
        else:
            y = tg.gemm_q2(x, twq, td, out_dtype=tg.OUT_BF16, workspace=ws)
            torch.cuda.synchronize()
            ref = oracle.q2_gemm(prob.x, wq_o, d_o, N)
    assert tg.device_error() == 0
    got = bf16_to_f32(bits16(y)).astype(np.float64)
    assert got.shape == (M, N)
    assert np.all(np.isfinite(got)), f"{name}: non-finite outputs"
    ref_bf16 = bf16_to_f32(oracle.f64_to_bf16(ref)).astype(np.float64)
    gate_full(got, ref_bf16, f"{name} at full size (all {M * N} outputs)")


def test_tiny_config_exact(oracle):
    """The tiny configuration as specified: 16 x 256 activations, 128 x 256 ternary weights,
    seed 0, f32 output, against the f64 oracle (no bf16 rounding of the result)."""
    w = synth.ALL["tiny"]
    assert (w.M, w.N, w.K, w.seed, w.out_f32) == (16, 128, 256, 0, True)
    prob = w.make()
    wq_o, d_o, twq, td = _packed_q2(oracle, prob)
    y = tg.gemm_q2(dev(prob.x, torch.bfloat16), twq, td, out_dtype=tg.OUT_F32)
    torch.cuda.synchronize()
    assert y.dtype == torch.float32 and tuple(y.shape) == (16, 128)
    ref = oracle.q2_gemm(prob.x, wq_o, d_o, w.N)
    gate(y.cpu().numpy().astype(np.float64), ref, "tiny configuration, f32 output")
    assert tg.device_error() == 0
