"""Full-size parity: every matmul of the benchmark step at its benchmark size (GPU).

Each workload runs exactly as bench.py launches it:
- the automatic path choice;
- the full workspace from tgemm_workspace_size, so the split-tile schedule is used where
  it is chosen;
- bf16 output;
- weights packed on the device.

The device pack must equal the oracle's pack byte for byte. Then about 2000 outputs are
drawn at random, plus the first and last rows and tokens and the tile edges. Each is
computed on its own by the oracle (f64) and the sample is held to the accuracy gates.
"""
import numpy as np
import pytest
import torch

import bit_weight_quantized_tgemm_b200 as tg
from bit_weight_quantized_tgemm_b200 import synth
from helpers import bf16_to_f32, bits16, dev, gate

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

STEP = ["mmdit_9216x3072", "mmdit_3072x12288", "mmdit_12288x3072", "lora_r4", "lora_r32",
        "lora_r64", "encoder_up", "encoder_down", "gemv_m1", "gemv_m4", "gemv_m16"]


def _sample(M, N, rng, n=2000):
    """Random (m, n) pairs plus the corners and the 128-row / 256-token tile edges."""
    mi = rng.integers(0, M, n)
    ni = rng.integers(0, N, n)
    edge_m = sorted({0, M - 1} | {t for t in range(255, M, 256)} | {t for t in range(256, M, 256)})
    edge_n = sorted({0, N - 1} | {t for t in range(127, N, 128 * 7)} | {t for t in range(128, N, 128 * 7)})
    em = np.array([m for m in edge_m for _ in edge_n], dtype=np.int64)
    en = np.array([c for _ in edge_m for c in edge_n], dtype=np.int64)
    return np.concatenate([mi, em]), np.concatenate([ni, en])


@pytest.fixture(autouse=True)
def auto_path():
    prev = tg.set_path(tg.PATH_AUTO)
    yield
    tg.set_path(prev)


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
    else:
        wq_o, d_o, st = oracle.q2_pack(prob.codes, prob.scale)
        assert st == 0
        twq, td, tst = tg.q2_pack(torch.from_numpy(prob.codes).cuda(), torch.from_numpy(prob.scale).cuda())
        torch.cuda.synchronize()
        assert int(tst.item()) == 0
        assert np.array_equal(twq.cpu().numpy(), wq_o), "device Q2 pack differs from the oracle"
        assert np.array_equal(bits16(td), d_o), "device scale pack differs from the oracle"
        if w.kind == "q2_lora":
            op, r = tg.OP_Q2_LORA, w.r
        else:
            op, r = tg.OP_Q2, 0
        ws = torch.empty(max(tg.workspace_size(op, M, N, K, r), 256), dtype=torch.uint8, device="cuda")
        if r:
            y = tg.gemm_q2_lora(x, twq, td, dev(prob.a, torch.bfloat16), dev(prob.b, torch.bfloat16),
                                out_dtype=tg.OUT_BF16, workspace=ws)
        else:
            y = tg.gemm_q2(x, twq, td, out_dtype=tg.OUT_BF16, workspace=ws)
    torch.cuda.synchronize()
    assert tg.device_error() == 0
    rng = np.random.default_rng(2024)
    mi, ni = _sample(M, N, rng)
    if w.kind == "q4":
        ref = oracle.q4_gemm_at(prob.x, wq_o, sz_o, N, mi, ni)
    elif w.kind == "q2_lora":
        ref = oracle.q2_gemm_at(prob.x, wq_o, d_o, N, mi, ni, prob.a, prob.b)
    else:
        ref = oracle.q2_gemm_at(prob.x, wq_o, d_o, N, mi, ni)
    ybits = bits16(y)
    got = bf16_to_f32(ybits[mi, ni]).astype(np.float64)
    assert np.all(np.isfinite(got))
    ref_bf16 = bf16_to_f32(oracle.f64_to_bf16(ref)).astype(np.float64)
    gate(got, ref_bf16, f"{name} at full size ({mi.size} sampled outputs)")
