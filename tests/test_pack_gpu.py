"""Device packing and dequantization against the oracle: bit-exact (GPU)."""
import numpy as np
import pytest
import torch

import bit_weight_quantized_tgemm_b200 as tg
from helpers import bits16, dev

pytestmark = pytest.mark.gpu


def _status(t):
    torch.cuda.synchronize()
    return int(t.item())


@pytest.mark.parametrize("N,K", [(1, 128), (37, 256), (128, 384), (300, 3072)])
def test_q2_pack_matches_oracle(oracle, N, K):
    rng = np.random.default_rng(N * 1000 + K)
    codes = rng.integers(0, 3, size=(N, K), dtype=np.uint8)
    scale = (np.abs(rng.standard_normal((N, K // 128))) * 0.02).astype(np.float16).astype(np.float32)
    wq, d, st = tg.q2_pack(dev(codes, torch.uint8), dev(scale, torch.float32))
    owq, od, ost = oracle.q2_pack(codes, scale)
    assert _status(st) == ost == 0
    assert np.array_equal(wq.cpu().numpy(), owq)
    assert np.array_equal(bits16(d), od)


def test_q2_pack_every_byte_and_status(oracle):
    # every byte value whose four codes are in {0,1,2} (81 of them), plus code 3 and > 3
    combos = np.array([[a, b, c, e] for a in range(3) for b in range(3) for c in range(3)
                       for e in range(3)], dtype=np.uint8)  # 81 x 4
    codes = np.ones((3, 384), dtype=np.uint8)
    codes[0, :324] = combos.reshape(-1)
    codes[1, 7] = 3
    codes[2, 100] = 200
    scale = np.array([[1.0, 0.5, 0.25], [0.02, 1.0, 1.0], [np.inf, 2.0, np.nan]], np.float32)
    wq, d, st = tg.q2_pack(dev(codes, torch.uint8), dev(scale, torch.float32))
    owq, od, ost = oracle.q2_pack(codes, scale)
    assert _status(st) == ost == (tg.PACK_BAD_CODE | tg.PACK_INEXACT | tg.PACK_NONFINITE)
    assert np.array_equal(wq.cpu().numpy(), owq)
    assert np.array_equal(bits16(d)[np.isfinite(scale)], od[np.isfinite(scale)])


def test_q2_pack_golden_bytes():
    rows = [l.split() for l in open(__file__.replace("test_pack_gpu.py", "golden/q2_bytes.txt"))
            if l.strip() and not l.startswith("#")]
    codes = np.ones((len(rows), 128), dtype=np.uint8)
    for i, r in enumerate(rows):
        codes[i, :4] = [int(v) for v in r[:4]]
    wq, _, st = tg.q2_pack(dev(codes, torch.uint8), dev(np.ones((len(rows), 1), np.float32), torch.float32))
    assert _status(st) == 0
    assert [int(v) for v in wq[:, 0].cpu()] == [int(r[4], 16) for r in rows]


def test_f16_scales_all_patterns(oracle):
    # every finite f16 value as an f32 scale must pack to its own bit pattern, status 0
    h = np.arange(65536, dtype=np.uint16)
    v = h.view(np.float16).astype(np.float32)
    fin = np.isfinite(v)
    vals = v[fin]
    hs = h[fin]
    n = (vals.size + 127) // 128 * 128
    scale = np.ones(n, np.float32)
    scale[: vals.size] = vals
    scale = scale.reshape(-1, 1)  # one block per row, K = 128
    codes = np.ones((scale.shape[0], 128), np.uint8)
    _, d, st = tg.q2_pack(dev(codes, torch.uint8), dev(scale, torch.float32))
    assert _status(st) == 0
    assert np.array_equal(bits16(d).reshape(-1)[: vals.size], hs)
    # and inexact values are flagged
    _, _, st = tg.q2_pack(dev(codes[:1], torch.uint8), dev(np.array([[0.02]], np.float32), torch.float32))
    assert _status(st) == tg.PACK_INEXACT


@pytest.mark.parametrize("N,K", [(1, 64), (29, 192), (256, 2560)])
def test_q4_pack_matches_oracle(oracle, N, K):
    rng = np.random.default_rng(N + K)
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    s = (np.abs(rng.standard_normal((N, K // 64))) * 0.01).astype(np.float16).astype(np.float32)
    z = rng.uniform(7, 8, size=(N, K // 64)).astype(np.float16).astype(np.float32)
    wq, sz, st = tg.q4_pack(dev(codes, torch.uint8), dev(s, torch.float32), dev(z, torch.float32))
    owq, osz, ost = oracle.q4_pack(codes, s, z)
    assert _status(st) == ost == 0
    assert np.array_equal(wq.cpu().numpy(), owq)
    assert np.array_equal(bits16(sz), osz)


def test_q4_pack_golden_and_status(oracle):
    rows = [l.split() for l in open(__file__.replace("test_pack_gpu.py", "golden/q4_bytes.txt"))
            if l.strip() and not l.startswith("#")]
    codes = np.zeros((len(rows) + 1, 64), dtype=np.uint8)
    for i, r in enumerate(rows):
        codes[i, 0], codes[i, 1] = int(r[0]), int(r[1])
    codes[-1, 5] = 16  # out of range
    one = np.ones((len(rows) + 1, 1), np.float32)
    z = one * 7.5
    z[0, 0] = 7.3  # not an f16 value
    wq, _, st = tg.q4_pack(dev(codes, torch.uint8), dev(one, torch.float32), dev(z, torch.float32))
    assert _status(st) == tg.PACK_BAD_CODE | tg.PACK_INEXACT
    got = wq[:, 0].cpu().numpy()
    assert [int(v) for v in got[: len(rows)]] == [int(r[2], 16) for r in rows]
    owq, _, _ = oracle.q4_pack(codes, one, z)
    assert np.array_equal(wq.cpu().numpy(), owq)


def test_q2_dequant_every_byte(oracle):
    wq = np.tile(np.arange(256, dtype=np.uint8), 4).reshape(8, 128)  # K = 512
    d = np.array([[1.0, -0.5, 0.02, 3.0]] * 8, np.float32).astype(np.float16).view(np.uint16)
    w = tg.q2_dequant(dev(wq, torch.uint8), dev(d, torch.float16))
    ow = oracle.q2_dequant(wq, d, 8, 512)
    assert np.array_equal(w.cpu().numpy().view(np.uint32), ow.view(np.uint32))


def test_q4_dequant_every_byte(oracle):
    rng = np.random.default_rng(3)
    wq = np.tile(np.arange(256, dtype=np.uint8), 2).reshape(4, 128)  # K = 256
    s = (np.abs(rng.standard_normal((4, 4))) * 0.01).astype(np.float16)
    z = rng.uniform(7, 8, size=(4, 4)).astype(np.float16)
    sz = np.stack([s, z], axis=-1).view(np.uint16)
    w = tg.q4_dequant(dev(wq, torch.uint8), dev(sz, torch.float16))
    ow = oracle.q4_dequant(wq, sz, 4, 256)
    assert np.array_equal(w.cpu().numpy().view(np.uint32), ow.view(np.uint32))
