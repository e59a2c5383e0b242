"""One MMDiT block pair's linears as a CUDA-graph-captured sequence (GPU).

The sequence is cut down to the text conditioning projection, one joint block and one
single block, at full width. Token counts are 200 image + 72 text, so M is ragged.
Weights come from the seeded generators and are packed by the oracle; every activation
buffer is filled from the same generators. The tests check that:
- replaying the captured graph gives bit for bit the outputs of the eager calls;
- every output of every linear passes the accuracy gates against the f64 oracle;
- linear1 run as two row-slice calls (pointer offsets into one packed matrix) agrees
  with the one-call result's columns.
"""
import numpy as np
import pytest
import torch

import bit_weight_quantized_tgemm_b200 as tg
from bit_weight_quantized_tgemm_b200 import mmdit, synth
from helpers import dev, gate_full, out_to_f64

pytestmark = pytest.mark.gpu

IMG, TXT = 200, 72


def _weights(oracle, shapes, seed):
    host, devw = {}, {}
    for i, name in enumerate(sorted(shapes)):
        n, k = shapes[name]
        p = synth.q2_problem((seed, i), 1, n, k)
        wq, d, st = oracle.q2_pack(p.codes, p.scale)
        assert st == 0
        host[name] = (wq, d)
        devw[name] = (dev(wq, torch.uint8), dev(d, torch.float16))
    return host, devw


def _fill_inputs(seq, seed):
    """Every activation buffer from the seeded generator; returns (M, K) -> bf16 bits."""
    host = {}
    for m, k in sorted(seq.inputs):
        bits = synth.q2_problem((seed, m, k), m, 1, k).x  # N(0, 1) activations as bf16
        seq.inputs[(m, k)].copy_(dev(bits, torch.bfloat16))
        host[(m, k)] = bits
    return host


@pytest.fixture(scope="module")
def step(oracle):
    shapes = mmdit.weight_shapes(joint_blocks=1, single_blocks=1)
    host_w, dev_w = _weights(oracle, shapes, 51)
    seq = mmdit.StepSequence(mmdit.step_linears(IMG, TXT, joint_blocks=1, single_blocks=1),
                             dev_w, out_dtype=tg.OUT_F32, distinct_outputs=True)
    host_x = _fill_inputs(seq, 52)
    return seq, host_w, host_x


def test_graph_replay_equals_eager(step):
    seq, _, _ = step
    seq.run()
    torch.cuda.synchronize()
    eager = [c.y.clone() for c in seq.calls]
    graph = seq.capture(warmup=1)
    for c in seq.calls:
        c.y.fill_(float("nan"))
    graph.replay()
    torch.cuda.synchronize()
    assert tg.device_error() == 0
    for c, ref in zip(seq.calls, eager):
        assert torch.equal(c.y, ref), f"{c.lin.name}: replay differs from the eager call"
    del graph


def test_every_linear_against_oracle(oracle, step):
    seq, host_w, host_x = step
    seq.run()
    torch.cuda.synchronize()
    for c in seq.calls:
        lin = c.lin
        wq, d = host_w[lin.weight]
        wq = wq[lin.row0:lin.row0 + lin.N]
        d = d[lin.row0:lin.row0 + lin.N]
        x = host_x[(lin.M, lin.K)]
        if lin.K2:
            wq2, d2 = host_w[lin.weight2]
            ref = oracle.q2_dual_gemm(x, wq, d, host_x[(lin.M, lin.K2)], wq2, d2, lin.N)
        else:
            ref = oracle.q2_gemm(x, wq, d, lin.N)
        # every output of the linear
        gate_full(out_to_f64(c.y), ref,
                  f"{lin.name} ({lin.M}x{lin.N}x{lin.K}{'+' + str(lin.K2) if lin.K2 else ''})")


def test_row_slices_match_stacked_call(step):
    seq, _, _ = step
    sliced = mmdit.StepSequence(
        mmdit.step_linears(IMG, TXT, joint_blocks=1, single_blocks=1, slice_rows=True),
        seq.weights, out_dtype=tg.OUT_F32, distinct_outputs=True)
    for key, buf in seq.inputs.items():
        sliced.inputs[key].copy_(buf)
    seq.run()
    sliced.run()
    torch.cuda.synchronize()
    whole = next(c.y for c in seq.calls if c.lin.name == "single0.linear1")
    qkv = next(c.y for c in sliced.calls if c.lin.name == "single0.linear1.qkv")
    up = next(c.y for c in sliced.calls if c.lin.name == "single0.linear1.mlp_up")
    for part, cols in ((qkv, slice(0, mmdit.QKV)), (up, slice(mmdit.QKV, None))):
        a, b = out_to_f64(part), out_to_f64(whole[:, cols].contiguous())
        rel = np.linalg.norm(a - b) / np.linalg.norm(b)
        assert rel < 1e-5, f"row slice differs from the stacked call by {rel:.2e}"
