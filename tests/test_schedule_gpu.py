"""Tensor-core schedules: tiles split between CTAs versus whole tiles per CTA (GPU).

Shapes whose tiles fill the SMs unevenly run with split tiles when the workspace has
room for the f32 partial sums (tgemm_workspace_size) and with whole tiles per CTA when
it holds only the minimum (tgemm_workspace_size_min).  Both must pass the accuracy gates
against the f64 oracle, agree with each other to f32 rounding, and the split schedule
must be deterministic (the partial sums are added in k order, whoever arrives last).
"""
import numpy as np
import pytest
import torch

import bit_weight_quantized_tgemm_b200 as tg
from bit_weight_quantized_tgemm_b200 import synth
from helpers import canary_intact, dev, gate, gate_output, nan_filled, out_to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def tensor_path():
    prev = tg.set_path(tg.PATH_TENSOR)
    yield
    tg.set_path(prev)


def _workspaces(op, M, N, K, r=0):
    full = tg.workspace_size(op, M, N, K, r)
    small = tg.workspace_size_min(op, M, N, K, r)
    assert full > small > 0, "this shape was chosen to run with split tiles"
    return (torch.empty(full, dtype=torch.uint8, device="cuda"),
            torch.empty(small, dtype=torch.uint8, device="cuda"))


def _both(run, M, N):
    """Run `run(workspace, y)` with the split and the whole-tile workspace (f32 out)."""
    outs = []
    for ws in run.workspaces:
        y, buf = nan_filled((M, N), torch.float32)
        run(ws, y)
        torch.cuda.synchronize()
        assert canary_intact(buf, M * N)
        outs.append(y)
    return outs


def _check(outs, ref, oracle, what):
    split, whole = outs
    gate_output(split, ref, oracle, what + " split tiles")
    gate_output(whole, ref, oracle, what + " whole tiles")
    a, b = out_to_f64(split), out_to_f64(whole)
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert rel < 1e-5, f"{what}: schedules differ by {rel:.2e}"


# Q2: 8 tiles of 32 stages (upc 2: every tile split 16 ways); 3 tiles of 64 stages with
# ragged token and row edges; and 2 x 8 tiles of 32 stages.
@pytest.mark.parametrize("M,N,K", [(256, 1024, 4096), (200, 300, 8192), (300, 1000, 4096)])
def test_q2_split_vs_whole(oracle, M, N, K):
    prob = synth.q2_problem((11, M, N, K), M, N, K)
    wq, d, st = oracle.q2_pack(prob.codes, prob.scale)
    assert st == 0
    x, twq, td = dev(prob.x, torch.bfloat16), dev(wq, torch.uint8), dev(d, torch.float16)

    def run(ws, y):
        tg.gemm_q2(x, twq, td, out_dtype=tg.OUT_F32, y=y, workspace=ws)
    run.workspaces = _workspaces(tg.OP_Q2, M, N, K)
    _check(_both(run, M, N), oracle.q2_gemm(prob.x, wq, d, N), oracle, f"q2 {M}x{N}x{K}")


# 4-bit: 2 x 10 tiles of 38 stages (the encoder's down projection, halved).
def test_q4_split_vs_whole(oracle):
    M, N, K = 512, 1280, 4864
    prob = synth.q4_problem((12, M, N, K), M, N, K)
    wq, sz, st = oracle.q4_pack(prob.codes, prob.s, prob.z)
    assert st == 0
    x, twq, tsz = dev(prob.x, torch.bfloat16), dev(wq, torch.uint8), dev(sz, torch.float16)

    def run(ws, y):
        tg.gemm_q4(x, twq, tsz, out_dtype=tg.OUT_F32, y=y, workspace=ws)
    run.workspaces = _workspaces(tg.OP_Q4, M, N, K)
    _check(_both(run, M, N), oracle.q4_gemm(prob.x, wq, sz, N), oracle, f"q4 {M}x{N}x{K}")


# Branch: 32 main + 1 branch stage per tile, upc 4, so the segment [32, 36) holds only
# tile 0's branch stage (the MMA must start that accumulator from zero).
@pytest.mark.parametrize("r", [4, 64])
def test_q2_lora_split_vs_whole(oracle, r):
    M, N, K = 300, 1000, 4096
    prob = synth.q2_problem((13, M, N, K, r), M, N, K, r=r)
    wq, d, st = oracle.q2_pack(prob.codes, prob.scale)
    assert st == 0
    x, twq, td = dev(prob.x, torch.bfloat16), dev(wq, torch.uint8), dev(d, torch.float16)
    a, b = dev(prob.a, torch.bfloat16), dev(prob.b, torch.bfloat16)

    def run(ws, y):
        tg.gemm_q2_lora(x, twq, td, a, b, out_dtype=tg.OUT_F32, y=y, workspace=ws)
    run.workspaces = _workspaces(tg.OP_Q2_LORA, M, N, K, r)
    _check(_both(run, M, N), oracle.q2_lora_gemm(prob.x, wq, d, prob.a, prob.b, N), oracle,
           f"q2+branch r={r}")


def test_split_is_deterministic(oracle):
    """Same inputs, three calls in a row (counters re-zeroed each call): identical bits."""
    M, N, K = 256, 1024, 4096
    prob = synth.q2_problem((14, M, N, K), M, N, K)
    wq, d, st = oracle.q2_pack(prob.codes, prob.scale)
    x, twq, td = dev(prob.x, torch.bfloat16), dev(wq, torch.uint8), dev(d, torch.float16)
    ws, _ = _workspaces(tg.OP_Q2, M, N, K)
    ys = [tg.gemm_q2(x, twq, td, out_dtype=tg.OUT_F32, workspace=ws) for _ in range(3)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(y, ys[0])
    assert tg.device_error() == 0


# ---- hybrid form: whole tiles first in the numbering, the remainder split over all CTAs
def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _sample(M, N, seed, n=1500):
    rng = np.random.default_rng(seed)
    mi = np.concatenate([rng.integers(0, M, n), [0, M - 1, 0, M - 1]]).astype(np.int64)
    ni = np.concatenate([rng.integers(0, N, n), [0, 0, N - 1, N - 1]]).astype(np.int64)
    return mi, ni


def _check_sampled(outs, ref_at, mi, ni, what):
    split, whole = outs
    ref = ref_at(mi, ni)
    for y, form in ((split, "hybrid"), (whole, "whole tiles")):
        gate(out_to_f64(y)[mi, ni], ref, f"{what} {form} ({mi.size} sampled outputs)")
    a, b = out_to_f64(split), out_to_f64(whole)
    assert np.all(np.isfinite(a)) and np.all(np.isfinite(b))
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert rel < 1e-5, f"{what}: schedules differ by {rel:.2e}"


def _hybrid(op, M, N, K, r=0, K2=0):
    pl = tg.tc_plan(op, M, N, K, r, K2, sms=_sms())
    assert pl["split"] and pl["dpc"] > 0, f"expected the hybrid form, got {pl}"
    return pl


# tiles: 200 (1 wave + 52), 2 x 104 with ragged token and row edges, 360 (the 1280-token QKV)
@pytest.mark.parametrize("M,N,K", [(256, 25600, 2048), (300, 13300, 3072), (1280, 9216, 3072)])
def test_q2_hybrid_vs_whole(oracle, M, N, K):
    _hybrid(tg.OP_Q2, M, N, K)
    prob = synth.q2_problem((21, M, N, K), M, N, K)
    wq, d, st = oracle.q2_pack(prob.codes, prob.scale)
    assert st == 0
    x, twq, td = dev(prob.x, torch.bfloat16), dev(wq, torch.uint8), dev(d, torch.float16)

    def run(ws, y):
        tg.gemm_q2(x, twq, td, out_dtype=tg.OUT_F32, y=y, workspace=ws)
    run.workspaces = _workspaces(tg.OP_Q2, M, N, K)
    mi, ni = _sample(M, N, 5)
    _check_sampled(_both(run, M, N), lambda a, b: oracle.q2_gemm_at(prob.x, wq, d, N, a, b),
                   mi, ni, f"q2 {M}x{N}x{K}")


def test_q4_hybrid_vs_whole(oracle):
    M, N, K = 512, 12800, 2048
    _hybrid(tg.OP_Q4, M, N, K)
    prob = synth.q4_problem((22, M, N, K), M, N, K)
    wq, sz, st = oracle.q4_pack(prob.codes, prob.s, prob.z)
    assert st == 0
    x, twq, tsz = dev(prob.x, torch.bfloat16), dev(wq, torch.uint8), dev(sz, torch.float16)

    def run(ws, y):
        tg.gemm_q4(x, twq, tsz, out_dtype=tg.OUT_F32, y=y, workspace=ws)
    run.workspaces = _workspaces(tg.OP_Q4, M, N, K)
    mi, ni = _sample(M, N, 6)
    _check_sampled(_both(run, M, N), lambda a, b: oracle.q4_gemm_at(prob.x, wq, sz, N, a, b),
                   mi, ni, f"q4 {M}x{N}x{K}")


@pytest.mark.parametrize("r", [4, 32])
def test_q2_lora_hybrid_vs_whole(oracle, r):
    M, N, K = 300, 13300, 3072
    _hybrid(tg.OP_Q2_LORA, M, N, K, r)
    prob = synth.q2_problem((23, M, N, K, r), M, N, K, r=r)
    wq, d, st = oracle.q2_pack(prob.codes, prob.scale)
    assert st == 0
    x, twq, td = dev(prob.x, torch.bfloat16), dev(wq, torch.uint8), dev(d, torch.float16)
    a, b = dev(prob.a, torch.bfloat16), dev(prob.b, torch.bfloat16)

    def run(ws, y):
        tg.gemm_q2_lora(x, twq, td, a, b, out_dtype=tg.OUT_F32, y=y, workspace=ws)
    run.workspaces = _workspaces(tg.OP_Q2_LORA, M, N, K, r)
    mi, ni = _sample(M, N, 7)
    _check_sampled(_both(run, M, N),
                   lambda i, j: oracle.q2_gemm_at(prob.x, wq, d, N, i, j, prob.a, prob.b),
                   mi, ni, f"q2+branch r={r} {M}x{N}x{K}")


def test_dual_hybrid_vs_whole(oracle):
    M, N, K1, K2 = 256, 25600, 1024, 1024
    _hybrid(tg.OP_Q2, M, N, K1, 0, K2)
    p1 = synth.q2_problem((24, 1), M, N, K1)
    p2 = synth.q2_problem((24, 2), M, N, K2)
    wq1, d1, s1 = oracle.q2_pack(p1.codes, p1.scale)
    wq2, d2, s2 = oracle.q2_pack(p2.codes, p2.scale)
    assert s1 == 0 and s2 == 0
    devs = (dev(p1.x, torch.bfloat16), dev(wq1, torch.uint8), dev(d1, torch.float16),
            dev(p2.x, torch.bfloat16), dev(wq2, torch.uint8), dev(d2, torch.float16))
    full = tg.dual_workspace_size(M, N, K1, K2)
    small = tg.dual_workspace_size(M, N, K1, K2, minimum=True)
    assert full > small > 0

    def run(ws, y):
        tg.gemm_q2_dual(*devs, out_dtype=tg.OUT_F32, y=y, workspace=ws)
    run.workspaces = (torch.empty(full, dtype=torch.uint8, device="cuda"),
                      torch.empty(small, dtype=torch.uint8, device="cuda"))
    mi, ni = _sample(M, N, 8)
    _check_sampled(_both(run, M, N),
                   lambda i, j: oracle.q2_dual_gemm_at(p1.x, wq1, d1, p2.x, wq2, d2, N, i, j),
                   mi, ni, f"dual {M}x{N}x({K1}+{K2})")


def test_hybrid_is_deterministic(oracle):
    M, N, K = 256, 25600, 2048
    _hybrid(tg.OP_Q2, M, N, K)
    prob = synth.q2_problem((25, M, N, K), M, N, K)
    wq, d, st = oracle.q2_pack(prob.codes, prob.scale)
    x, twq, td = dev(prob.x, torch.bfloat16), dev(wq, torch.uint8), dev(d, torch.float16)
    ws, _ = _workspaces(tg.OP_Q2, M, N, K)
    ys = [tg.gemm_q2(x, twq, td, out_dtype=tg.OUT_F32, workspace=ws) for _ in range(3)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(y, ys[0])
    assert tg.device_error() == 0
