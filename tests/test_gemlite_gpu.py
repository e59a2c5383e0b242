"""gemlite-int2 -> Q2_0 import on the device against the oracle's import (GPU).

The gemlite representation is built here from seeded codes and scales. Its bytes are
[K/4][N], byte (i, n) holding the codes of k = 4i..4i+3 of row n, LSB-first. Scale and
zero are f32 [N][K/g] with zero = -scale. The device import must equal the oracle's
byte for byte (wq, d) and report the same status bits. A matmul on the imported weights
then passes the accuracy gates against the oracle.
"""
import numpy as np
import pytest
import torch

import bit_weight_quantized_tgemm_b200 as tg
from bit_weight_quantized_tgemm_b200 import synth
from helpers import bits16, dev, gate_output

pytestmark = pytest.mark.gpu


def gemlite_problem(seed: int, N, K, g):
    """Seeded codes and per-128-block scales, expressed in the gemlite layout."""
    p = synth.q2_problem((seed, N, K, g), 1, N, K)
    c = p.codes.T.reshape(K // 4, 4, N).astype(np.uint32)
    wq_g = (c[:, 0] | (c[:, 1] << 2) | (c[:, 2] << 4) | (c[:, 3] << 6)).astype(np.uint8)
    if g <= 128:
        scale = np.repeat(p.scale, 128 // g, axis=1)
    else:
        rng = np.random.default_rng((seed, 7, g))
        scale = np.abs(rng.standard_normal((N, K // g)) * 0.02).astype(np.float16).astype(np.float32)
    return p, np.ascontiguousarray(wq_g), np.ascontiguousarray(scale, np.float32)


def _device_import(wq_g, scale, zero, g):
    wq, d, st = tg.q2_from_gemlite(torch.from_numpy(wq_g).cuda(), torch.from_numpy(scale).cuda(),
                                   torch.from_numpy(zero).cuda(), g)
    torch.cuda.synchronize()
    return wq.cpu().numpy(), bits16(d), int(st.item())


@pytest.mark.parametrize("N,K,g", [(1, 128, 128), (130, 256, 64), (300, 1024, 32), (64, 512, 256),
                                   (257, 3072, 3072), (1000, 1536, 128), (129, 384, 4)])
def test_import_matches_oracle(oracle, N, K, g):
    _, wq_g, scale = gemlite_problem(61, N, K, g)
    zero = -scale
    want = oracle.q2_from_gemlite(wq_g, scale, zero, g)
    assert want[2] == 0
    wq, d, st = _device_import(wq_g, scale, zero, g)
    assert st == 0
    assert np.array_equal(wq, want[0]), "packed bytes differ from the oracle's import"
    assert np.array_equal(d, want[1]), "block scales differ from the oracle's import"


def test_import_status_matches_oracle(oracle):
    N, K, g = 70, 512, 64
    _, wq_g, scale = gemlite_problem(62, N, K, g)
    zero = -scale
    cases = []
    z = zero.copy()
    z[3, 5] = 1.0
    cases.append(("zero mismatch", wq_g, scale, z, tg.PACK_ZERO_MISMATCH))
    s = scale.copy()
    s[69, 7] = s[69, 6] * 2
    cases.append(("group mismatch", wq_g, s, -s, tg.PACK_GROUP_MISMATCH))
    bad = wq_g.copy()
    bad[100, 33] |= 0x30
    cases.append(("code 3", bad, scale, zero, tg.PACK_BAD_CODE))
    s = scale.copy()
    s[0, 0:2] = np.float32(0.02)
    cases.append(("inexact scale", wq_g, s, -s, tg.PACK_INEXACT))
    s = scale.copy()
    s[5, 2:4] = np.inf
    cases.append(("infinite scale", wq_g, s, -s, tg.PACK_NONFINITE))
    for what, a, b, c, bit in cases:
        want = oracle.q2_from_gemlite(a, b, c, g)
        got = _device_import(a, b, c, g)
        assert want[2] & bit, what
        assert got[2] == want[2], f"{what}: status {got[2]} != oracle {want[2]}"
        assert np.array_equal(got[0], want[0]), what


def test_imported_weights_in_matmul(oracle):
    """Import on the device, then y = x W^T on both paths against the oracle."""
    N, K, g = 300, 1024, 64
    p, wq_g, scale = gemlite_problem(63, N, K, g)
    wq_o, d_o, st = oracle.q2_from_gemlite(wq_g, scale, -scale, g)
    assert st == 0
    wq, d, st = tg.q2_from_gemlite(torch.from_numpy(wq_g).cuda(), torch.from_numpy(scale).cuda(),
                                   torch.from_numpy(-scale).cuda(), g)
    assert int(st.item()) == 0
    prev = tg.set_path(tg.PATH_AUTO)
    try:
        for M in (1, 7, 200):
            x = synth.q2_problem((64, M), M, 1, K).x
            y = tg.gemm_q2(dev(x, torch.bfloat16), wq, d, out_dtype=tg.OUT_F32)
            torch.cuda.synchronize()
            gate_output(y, oracle.q2_gemm(x, wq_o, d_o, N), oracle, f"imported weights, M={M}")
    finally:
        tg.set_path(prev)


@pytest.mark.slow
def test_import_mmdit_qkv_full_size(oracle):
    """The MMDiT's 9216 x 3072 qkv matrix with one group per block: byte-exact."""
    N, K, g = 9216, 3072, 128
    _, wq_g, scale = gemlite_problem(65, N, K, g)
    want = oracle.q2_from_gemlite(wq_g, scale, -scale, g)
    got = _device_import(wq_g, scale, -scale, g)
    assert want[2] == 0 and got[2] == 0
    assert np.array_equal(got[0], want[0]) and np.array_equal(got[1], want[1])
