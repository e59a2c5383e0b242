"""Two matmuls at once on two streams (GPU).

No CTA of any kernel waits for another CTA: a tile shared by several CTAs (split tiles of
the tensor-core kernel) is finished by whichever sharer arrives last, so a grid needs no
guarantee that all its CTAs are resident at once.  Here two all-split grids (the text
encoder's up projection, 512 tokens x 9728 x 2560, each on its own stream and workspace)
run at the same time, next to a Q2 matmul on a third stream.  Each must match the oracle, the device error
word must stay clear (no wait ran out), and the whole must finish far below the 1 s wait
limit.
"""
import time

import numpy as np
import pytest
import torch

import bit_weight_quantized_tgemm_b200 as tg
from bit_weight_quantized_tgemm_b200 import synth
from helpers import bf16_to_f32, bits16, dev, gate_full

pytestmark = pytest.mark.gpu


def test_two_split_4bit_matmuls_on_two_streams(oracle):
    prev = tg.set_path(tg.PATH_AUTO)
    try:
        M, N, K = 512, 9728, 2560
        plan = tg.tc_plan(tg.OP_Q4, M, N, K, sms=torch.cuda.get_device_properties(0).multi_processor_count)
        assert plan["split"] == 1 and plan["dpc"] == 0  # every tile split
        probs = [synth.q4_problem((71, i), M, N, K) for i in range(2)]
        packed = [oracle.q4_pack(p.codes, p.s, p.z) for p in probs]
        xs = [dev(p.x, torch.bfloat16) for p in probs]
        ws = [dev(wq, torch.uint8) for wq, _, _ in packed]
        szs = [dev(sz, torch.float16) for _, sz, _ in packed]
        ys = [torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
        wss = [torch.empty(tg.workspace_size(tg.OP_Q4, M, N, K), dtype=torch.uint8, device="cuda")
               for _ in range(2)]
        q2 = synth.q2_problem(72, 1536, 3072, 3072)
        q2wq, q2d, _ = oracle.q2_pack(q2.codes, q2.scale)
        q2x, q2w, q2dd = dev(q2.x, torch.bfloat16), dev(q2wq, torch.uint8), dev(q2d, torch.float16)
        streams = [torch.cuda.Stream() for _ in range(3)]
        torch.cuda.synchronize()
        t0 = time.monotonic()
        for rep in range(3):
            for i in range(2):
                with torch.cuda.stream(streams[i]):
                    tg.gemm_q4(xs[i], ws[i], szs[i], out_dtype=tg.OUT_BF16, y=ys[i], workspace=wss[i])
            with torch.cuda.stream(streams[2]):
                yq2 = tg.gemm_q2(q2x, q2w, q2dd, out_dtype=tg.OUT_BF16)
        torch.cuda.synchronize()
        elapsed = time.monotonic() - t0
        assert tg.device_error() == 0, "a bounded wait ran out"
        assert elapsed < 0.5, f"concurrent calls took {elapsed:.3f} s"
        for i in range(2):
            wq, sz, _ = packed[i]
            ref = oracle.q4_gemm(probs[i].x, wq, sz, N)
            gate_full(bf16_to_f32(bits16(ys[i])).astype(np.float64),
                      bf16_to_f32(oracle.f64_to_bf16(ref)).astype(np.float64), f"stream {i}")
        ref = oracle.q2_gemm(q2.x, q2wq, q2d, 3072)
        gate_full(bf16_to_f32(bits16(yq2)).astype(np.float64),
                  bf16_to_f32(oracle.f64_to_bf16(ref)).astype(np.float64), "Q2 next to them")
    finally:
        tg.set_path(prev)
