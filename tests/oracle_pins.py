"""Pins that tie the CPU oracle to what the pages and plain mathematics fix.

Each ``pin_*`` function takes an :class:`oracle.Oracle` and raises ``AssertionError`` if
the oracle disagrees with something that does not come from the oracle itself: bytes
worked out by hand from the pages' rules (``tests/golden``), library conversions
(numpy's float16, torch's bfloat16), closed forms, invariants, and brute force along a
different algebraic route.  ``test_oracle.py`` runs them on the real oracle;
``test_oracle_mutants.py`` runs them on oracle builds with one planted mistake each and
checks that at least one pin fails.
"""
from __future__ import annotations

import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rows(name):
    out = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                out.append(line.split())
    return out


def _bf16(a):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def _bf16_f32(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


def _f16_bits(v):
    return np.asarray(v, dtype=np.float32).astype(np.float16).view(np.uint16)


# ---- Q2_0 packing: hand-built bytes ---------------------------------------------------

def pin_q2_hand_bytes(o):
    """Codes -> bytes worked by hand from the LSB-first rule; MSB-first is rejected."""
    rows = _rows("q2_bytes.txt")
    codes = np.array([[int(c) for c in r[:4]] for r in rows], dtype=np.uint8)
    want = np.array([int(r[4], 16) for r in rows], dtype=np.uint8)
    msb = np.array([int(r[5], 16) for r in rows], dtype=np.uint8)
    n = len(rows)
    # pack one row of K = 128 whose first four codes are the hand-built ones
    full = np.ones((n, 128), dtype=np.uint8)
    full[:, :4] = codes
    wq, d, st = o.q2_pack(full, np.ones((n, 1), dtype=np.float32))
    assert st == 0, st
    assert np.array_equal(wq[:, 0], want), (wq[:, 0], want)
    differs = want != msb
    assert not np.any(wq[differs, 0] == msb[differs])
    # all-ones codes pack to 0x55 in every other byte
    assert np.all(wq[:, 1:] == 0x55)
    # unpack reverses it
    back = o.q2_unpack(wq, n, 128)
    assert np.array_equal(back, full)


def pin_q2_exhaustive_roundtrip(o):
    """Every byte whose four codes are in {0,1,2} survives unpack -> pack unchanged."""
    allb = np.arange(256, dtype=np.uint8)
    wq = allb.reshape(8, 32)  # 8 rows x 32 bytes = every byte value once
    codes = o.q2_unpack(wq, 8, 128)
    assert codes.max() <= 3
    ok = (codes.reshape(8, 32, 4) <= 2).all(axis=2)
    wq2, _, st = o.q2_pack(np.minimum(codes, 2), np.ones((8, 1), dtype=np.float32))
    assert np.array_equal(wq2[ok], wq[ok])
    # the count of bytes without code 3 is 3^4
    assert int(ok.sum()) == 81


def pin_q2_ternary_values(o):
    """(q - 1) d takes only the values -d, 0, +d; code 1 gives exactly 0."""
    rng = np.random.default_rng(7)
    N, K = 6, 256
    codes = rng.integers(0, 3, size=(N, K), dtype=np.uint8)
    scale = np.abs(rng.standard_normal((N, K // 128)).astype(np.float32)) * 0.02
    scale = scale.astype(np.float16).astype(np.float32)
    wq, d, st = o.q2_pack(codes, scale)
    assert st == 0
    w = o.q2_dequant(wq, d, N, K)
    dd = np.repeat(scale, 128, axis=1)
    assert np.array_equal(w[codes == 0], -dd[codes == 0])
    assert np.array_equal(w[codes == 2], dd[codes == 2])
    assert np.all(w[codes == 1] == 0.0)


def pin_q2_scale_block(o):
    """Each 128-weight block along K uses its own scale (block b covers k in [128b, 128b+128))."""
    N, K = 1, 512
    codes = np.full((N, K), 2, dtype=np.uint8)
    scale = np.array([[1.0, 2.0, 4.0, 8.0]], dtype=np.float32)
    wq, d, _ = o.q2_pack(codes, scale)
    w = o.q2_dequant(wq, d, N, K)
    want = np.repeat(scale, 128, axis=1)
    assert np.array_equal(w, want)


# ---- 4-bit packing: hand-built bytes --------------------------------------------------

def pin_q4_hand_bytes(o):
    """(even, odd) codes -> byte with the even index in the low nibble; inverted select rejected."""
    rows = _rows("q4_bytes.txt")
    n = len(rows)
    full = np.zeros((n, 64), dtype=np.uint8)
    full[:, 0] = [int(r[0]) for r in rows]
    full[:, 1] = [int(r[1]) for r in rows]
    want = np.array([int(r[2], 16) for r in rows], dtype=np.uint8)
    inv = np.array([int(r[3], 16) for r in rows], dtype=np.uint8)
    one = np.ones((n, 1), dtype=np.float32)
    wq, sz, st = o.q4_pack(full, one, 0 * one)
    assert st == 0
    assert np.array_equal(wq[:, 0], want), (wq[:, 0], want)
    differs = want != inv
    assert not np.any(wq[differs, 0] == inv[differs])
    back = o.q4_unpack(wq, n, 64)
    assert np.array_equal(back, full)


def pin_q4_two_column_matmul(o):
    """The pages' tiny 2-column matmul (hand-worked values in golden/q4_two_column.txt)."""
    (row,) = _rows("q4_two_column.txt")
    x0, x1, c00, c01, c10, c11, y0, y1, sy0, sy1 = (int(v) for v in row)
    K = 64
    x = np.zeros((1, K), dtype=np.float32)
    x[0, 0], x[0, 1] = x0, x1
    codes = np.zeros((2, K), dtype=np.uint8)
    codes[0, 0], codes[0, 1], codes[1, 0], codes[1, 1] = c00, c01, c10, c11
    one = np.ones((2, 1), dtype=np.float32)
    wq, sz, _ = o.q4_pack(codes, one, 0 * one)
    y = o.q4_gemm(_bf16(x), wq, sz, 2)
    assert y[0, 0] == y0 and y[0, 1] == y1, (y, (y0, y1), (sy0, sy1))


def pin_q4_exhaustive_roundtrip(o):
    allb = np.arange(256, dtype=np.uint8).reshape(8, 32)
    codes = o.q4_unpack(allb, 8, 64)
    wq, _, st = o.q4_pack(codes, np.ones((8, 1), np.float32), np.zeros((8, 1), np.float32))
    assert st == 0
    assert np.array_equal(wq, allb)


def pin_q4_integer_weights(o):
    """s = 1, z = 0 gives w = q; s = 1, z = 8 gives w = q - 8: products with an integer matrix."""
    rng = np.random.default_rng(11)
    M, N, K = 5, 7, 128
    xi = rng.integers(-4, 5, size=(M, K)).astype(np.float32)  # exact in bf16
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    for zval in (0.0, 8.0):
        wq, sz, st = o.q4_pack(codes, np.ones((N, K // 64), np.float32),
                               np.full((N, K // 64), zval, np.float32))
        assert st == 0
        y = o.q4_gemm(_bf16(xi), wq, sz, N)
        want = xi.astype(np.int64) @ (codes.astype(np.int64) - int(zval)).T
        assert np.array_equal(y, want.astype(np.float64))


def pin_q4_dequant_groups(o):
    """Group g of 64 weights along K uses its own (s, z); w = (q - z) s."""
    N, K = 1, 192
    codes = np.full((N, K), 9, dtype=np.uint8)
    s = np.array([[0.5, 2.0, 0.25]], np.float32)
    z = np.array([[7.5, 7.0, 8.0]], np.float32)
    wq, sz, st = o.q4_pack(codes, s, z)
    assert st == 0
    w = o.q4_dequant(wq, sz, N, K)
    want = np.repeat(np.array([[0.75, 4.0, 0.25]], np.float32), 64, axis=1)
    assert np.array_equal(w, want)


# ---- scale conversions -----------------------------------------------------------------

def pin_f16_all_patterns(o):
    """f16 -> f32 matches numpy for all 65536 patterns; f32 -> f16 round-trips every finite one."""
    bad = 0
    for h in range(65536):
        ref = np.array([h], dtype=np.uint16).view(np.float16).astype(np.float32)[0]
        got = o.f16_to_f32(h)
        if np.isnan(ref):
            bad += not np.isnan(got)
            continue
        bad += not (got == ref and np.signbit(got) == np.signbit(ref))
        bad += o.f32_to_f16(float(ref)) != h
    assert bad == 0, bad


def pin_f32_to_f16_rounding(o):
    """Round to nearest even against numpy on random, tie, subnormal and overflow inputs."""
    rng = np.random.default_rng(3)
    vals = [rng.standard_normal(4000).astype(np.float32) * 0.02,
            rng.standard_normal(2000).astype(np.float32) * 3000.0,
            (rng.standard_normal(2000) * 1e-6).astype(np.float32)]
    # exact midpoints between neighbouring f16 values (ties)
    h = rng.integers(0, 0x7BFF, size=2000).astype(np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    vals.append(((lo + hi) / 2).astype(np.float32))
    vals.append(np.array([65504.0, 65519.0, 65520.0, 65536.0, 1e-8, 2.0 ** -25,
                          2.0 ** -24, 3 * 2.0 ** -26], dtype=np.float32))
    v = np.concatenate(vals)
    with np.errstate(over="ignore"):
        want = v.astype(np.float16).view(np.uint16)
    got = np.array([o.f32_to_f16(float(t)) for t in v], dtype=np.uint16)
    assert np.array_equal(got, want), np.flatnonzero(got != want)[:10]


def pin_bf16_rounding(o):
    """f32 -> bf16 matches torch (nearest even); f64 -> bf16 picks the nearest, ties to even."""
    import torch

    rng = np.random.default_rng(5)
    v = np.concatenate([rng.standard_normal(5000).astype(np.float32) * 10,
                        (rng.integers(0, 1 << 30, 2000).astype(np.uint32) | 0x8000)
                        .view(np.float32)])  # many exact ties in the low half
    v = v[np.isfinite(v)]
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([o.f32_to_bf16(float(t)) for t in v], dtype=np.uint16)
    assert np.array_equal(got, want)
    # f64 -> bf16: compare with exact rational nearest-even rounding
    d = np.concatenate([rng.standard_normal(3000) * 7.0, [0.5 + 2.0 ** -9, 1.0 + 2.0 ** -8,
                                                          1.0 + 3 * 2.0 ** -8, -2.5]])
    got = o.f64_to_bf16(d)
    for val, g in zip(d, got):
        gv = Fraction(float(_bf16_f32(np.array([g]))[0]))
        fv = Fraction(float(val))
        # neighbours of g in bf16
        up = Fraction(float(_bf16_f32(np.array([g + 1]))[0]))
        dn = Fraction(float(_bf16_f32(np.array([g - 1]))[0])) if g & 0x7FFF else -up
        assert abs(fv - gv) <= abs(fv - up) and abs(fv - gv) <= abs(fv - dn)
        if abs(fv - gv) == abs(fv - up) or abs(fv - gv) == abs(fv - dn):
            assert (int(g) & 1) == 0  # tie -> even significand


def pin_pack_status(o):
    """Inexact scale (0.02 is not an f16 value), code 3 and non-finite scales are flagged."""
    codes = np.ones((1, 128), dtype=np.uint8)
    _, d, st = o.q2_pack(codes, np.array([[0.02]], np.float32))
    assert st == 2
    exact = float(np.float32(np.float16(0.02)))
    _, d, st = o.q2_pack(codes, np.array([[exact]], np.float32))
    assert st == 0 and o.f16_to_f32(int(d[0, 0])) == exact
    c3 = codes.copy()
    c3[0, 5] = 3
    _, _, st = o.q2_pack(c3, np.array([[1.0]], np.float32))
    assert st == 1
    _, _, st = o.q2_pack(codes, np.array([[np.inf]], np.float32))
    assert st == 4
    c4 = np.zeros((1, 64), dtype=np.uint8)
    c4[0, 3] = 16
    _, _, st = o.q4_pack(c4, np.ones((1, 1), np.float32), np.zeros((1, 1), np.float32))
    assert st == 1
    _, _, st = o.q4_pack(c4 * 0, np.ones((1, 1), np.float32), np.full((1, 1), 7.3, np.float32))
    assert st == 2


# ---- gemlite-int2 import ----------------------------------------------------------------

def _gemlite_from_rows(rows):
    N, K = 2, 128
    wq_g = np.full((K // 4, N), 0x55, dtype=np.uint8)
    scale = np.zeros((N, 1), np.float32)
    zero = np.zeros((N, 1), np.float32)
    d_want = np.zeros((N, 1), np.uint16)
    w_want = []
    for r in rows:
        if r[0] == "byte":
            wq_g[int(r[1]), int(r[2])] = int(r[3], 16)
        elif r[0] == "scale":
            n = int(r[1])
            scale[n, 0], zero[n, 0], d_want[n, 0] = float(r[2]), float(r[3]), int(r[4], 16)
        elif r[0] == "w":
            w_want.append((int(r[1]), int(r[2]), float(r[3])))
    return wq_g, scale, zero, d_want, w_want


def pin_gemlite_hand_example(o):
    """A hand-worked import: each gemlite byte (i, n) becomes Q2_0 byte (n, i) unchanged,
    the scales become f16 d, and the dequantized weights are the hand-computed ones."""
    wq_g, scale, zero, d_want, w_want = _gemlite_from_rows(_rows("gemlite_small.txt"))
    wq, d, st = o.q2_from_gemlite(wq_g, scale, zero, 128)
    assert st == 0, st
    assert np.array_equal(wq, wq_g.T), "the import is a transpose of the packed bytes"
    assert np.array_equal(d, d_want)
    w = o.q2_dequant(wq, d, 2, 128)
    for n, k, v in w_want:
        assert w[n, k] == v, (n, k, w[n, k], v)


def _gemlite_random(rng, N, K, g):
    codes = rng.integers(0, 3, size=(N, K), dtype=np.uint8)
    # gemlite bytes [K/4][N]: byte (i, n) = sum_j codes[n][4i + j] << 2j
    c = codes.T.reshape(K // 4, 4, N).astype(np.uint32)
    wq_g = (c[:, 0] | (c[:, 1] << 2) | (c[:, 2] << 4) | (c[:, 3] << 6)).astype(np.uint8)
    per_block = np.abs(rng.standard_normal((N, K // 128))).astype(np.float16).astype(np.float32)
    if g <= 128:
        scale = np.repeat(per_block, 128 // g, axis=1)  # groups inside a block agree
    else:
        scale = np.abs(rng.standard_normal((N, K // g))).astype(np.float16).astype(np.float32)
    return codes, wq_g, scale, -scale


def pin_gemlite_dequant_definition(o):
    """For every group size, Q2_0 dequant of the import equals gemlite's own definition
    q * scale + zero evaluated from the gemlite bytes (exactly: both are one f32 product)."""
    rng = np.random.default_rng(90)
    N, K = 6, 1024
    for g in (32, 64, 128, 256, 512, 1024):
        codes, wq_g, scale, zero = _gemlite_random(rng, N, K, g)
        wq, d, st = o.q2_from_gemlite(wq_g, scale, zero, g)
        assert st == 0, (g, st)
        # gemlite's dequant, from its bytes: the code of (n, k) is in byte (k / 4, n)
        k = np.arange(K)
        q = (wq_g[k // 4, :] >> (2 * (k % 4))[:, None]) & 3          # [K][N]
        w_g = q.T.astype(np.float32) * np.repeat(scale, g, axis=1) + np.repeat(zero, g, axis=1)
        assert np.array_equal(q.T, codes)
        assert np.array_equal(o.q2_dequant(wq, d, N, K), w_g), g


def pin_gemlite_status(o):
    """zero != -scale, disagreeing groups in one block, a code 3 and an inexact f16 scale
    are each reported; a clean import reports nothing."""
    rng = np.random.default_rng(91)
    N, K = 3, 256
    codes, wq_g, scale, zero = _gemlite_random(rng, N, K, 64)
    assert o.q2_from_gemlite(wq_g, scale, zero, 64)[2] == 0
    z = zero.copy()
    z[1, 2] = -z[1, 2]
    if z[1, 2] == zero[1, 2]:
        z[1, 2] = 1.0
    assert o.q2_from_gemlite(wq_g, scale, z, 64)[2] == 8
    s = scale.copy()
    s[2, 1] = s[2, 0] * 2  # groups 0 and 1 form block 0 of row 2
    assert o.q2_from_gemlite(wq_g, s, -s, 64)[2] == 16
    bad = wq_g.copy()
    bad[5, 1] |= 0x0C  # code 3 at k = 21 of row 1
    assert o.q2_from_gemlite(bad, scale, zero, 64)[2] == 1
    s = scale.copy()
    s[0, :2] = np.float32(0.02)  # not an f16 value
    assert o.q2_from_gemlite(wq_g, s, -s, 64)[2] == 2


# ---- matmul: closed forms and brute force ---------------------------------------------

def _rand_x(rng, M, K, scale=1.0):
    return _bf16(rng.standard_normal((M, K)).astype(np.float32) * scale)


def pin_q2_matmul_closed_forms(o):
    rng = np.random.default_rng(13)
    M, N, K = 4, 6, 256
    x = _rand_x(rng, M, K)
    xf = _bf16_f32(x).astype(np.float64)
    one = np.ones((N, K // 128), np.float32)
    # all codes 1 -> y == 0 exactly
    wq, d, _ = o.q2_pack(np.ones((N, K), np.uint8), one)
    assert np.all(o.q2_gemm(x, wq, d, N) == 0.0)
    # all codes 2, d = 1 -> row sums of x in every column
    wq, d, _ = o.q2_pack(np.full((N, K), 2, np.uint8), one)
    y = o.q2_gemm(x, wq, d, N)
    assert np.allclose(y, np.repeat(xf.sum(axis=1, keepdims=True), N, axis=1), rtol=1e-12,
                       atol=1e-12)
    # one-hot code 2 at (n0, k0), code 0 at (n1, k1), else 1 -> y[:, n0] = d x[:, k0], y[:, n1] = -d x[:, k1]
    codes = np.ones((N, K), np.uint8)
    codes[2, 77] = 2
    codes[4, 200] = 0
    sc = np.full((N, K // 128), 0.25, np.float32)
    wq, d, _ = o.q2_pack(codes, sc)
    y = o.q2_gemm(x, wq, d, N)
    want = np.zeros((M, N))
    want[:, 2] = 0.25 * xf[:, 77]
    want[:, 4] = -0.25 * xf[:, 200]
    assert np.array_equal(y, want)


def pin_q2_matmul_brute_force(o):
    """Tiny shapes against the sign-sum form sum_b d_b (sum_{q=2} x - sum_{q=0} x), exact in Fraction."""
    for seed in range(10):
        rng = np.random.default_rng(100 + seed)
        M, N = int(rng.integers(1, 9)), int(rng.integers(1, 9))
        K = int(rng.choice([128, 256]))
        x = _rand_x(rng, M, K)
        xf = _bf16_f32(x)
        codes = rng.integers(0, 3, size=(N, K), dtype=np.uint8)
        sc = np.abs(rng.standard_normal((N, K // 128))).astype(np.float16).astype(np.float32)
        wq, d, st = o.q2_pack(codes, sc)
        assert st == 0
        y = o.q2_gemm(x, wq, d, N)
        for m in range(M):
            for n in range(N):
                tot = Fraction(0)
                for b in range(K // 128):
                    blk = slice(128 * b, 128 * (b + 1))
                    pos = sum(Fraction(float(v)) for v in xf[m, blk][codes[n, blk] == 2])
                    neg = sum(Fraction(float(v)) for v in xf[m, blk][codes[n, blk] == 0])
                    tot += Fraction(float(sc[n, b])) * (pos - neg)
                err = abs(Fraction(float(y[m, n])) - tot)
                assert err <= Fraction(1, 10 ** 9) * (1 + abs(tot)), (seed, m, n, float(err))


def pin_q4_matmul_brute_force(o):
    """Tiny shapes against sum_g s_g (sum q x - z sum x) in Fraction arithmetic."""
    for seed in range(6):
        rng = np.random.default_rng(200 + seed)
        M, N = int(rng.integers(1, 6)), int(rng.integers(1, 6))
        K = int(rng.choice([64, 128, 192]))
        x = _rand_x(rng, M, K)
        xf = _bf16_f32(x)
        codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
        s = (np.abs(rng.standard_normal((N, K // 64))) * 0.01).astype(np.float16).astype(np.float32)
        z = rng.uniform(7, 8, size=(N, K // 64)).astype(np.float16).astype(np.float32)
        wq, sz, st = o.q4_pack(codes, s, z)
        assert st == 0
        y = o.q4_gemm(x, wq, sz, N)
        for m in range(M):
            for n in range(N):
                tot = Fraction(0)
                for g in range(K // 64):
                    blk = slice(64 * g, 64 * (g + 1))
                    qx = sum(Fraction(int(q)) * Fraction(float(v))
                             for q, v in zip(codes[n, blk], xf[m, blk]))
                    sx = sum(Fraction(float(v)) for v in xf[m, blk])
                    tot += Fraction(float(s[n, g])) * (qx - Fraction(float(z[n, g])) * sx)
                # the oracle rounds w = (q - z) s to f32 first: allow that rounding
                bound = Fraction(1, 10 ** 5) * (1 + abs(tot))
                assert abs(Fraction(float(y[m, n])) - tot) <= bound, (seed, m, n)


def pin_square_matmul_orientation(o):
    """y[m, n] pairs row n of W with row m of x (a transposed W gives a different answer)."""
    N = K = 128
    codes = np.ones((N, K), np.uint8)
    codes[3, 90] = 2  # only W[3, 90] is nonzero
    wq, d, _ = o.q2_pack(codes, np.ones((N, 1), np.float32))
    x = np.zeros((2, K), np.float32)
    x[0, 90] = 5.0
    x[1, 3] = 7.0
    y = o.q2_gemm(_bf16(x), wq, d, N)
    want = np.zeros((2, N))
    want[0, 3] = 5.0
    assert np.array_equal(y, want)


def pin_lora_branch(o):
    """W == 0 leaves y = B (A x), checked against numpy's f64 matmul; and the branch adds linearly."""
    rng = np.random.default_rng(17)
    M, N, K, r = 5, 9, 128, 4
    x = _rand_x(rng, M, K)
    a = _rand_x(rng, r, K)
    b = _rand_x(rng, N, r)
    wq, d, _ = o.q2_pack(np.ones((N, K), np.uint8), np.ones((N, 1), np.float32))
    y = o.q2_lora_gemm(x, wq, d, a, b, N)
    xf, af, bf = (_bf16_f32(t).astype(np.float64) for t in (x, a, b))
    want = (xf @ af.T) @ bf.T
    assert np.allclose(y, want, rtol=1e-12, atol=1e-12)
    # with a real W: branch = lora_gemm - gemm
    codes = rng.integers(0, 3, size=(N, K), dtype=np.uint8)
    wq, d, _ = o.q2_pack(codes, np.full((N, 1), 0.5, np.float32))
    diff = o.q2_lora_gemm(x, wq, d, a, b, N) - o.q2_gemm(x, wq, d, N)
    assert np.allclose(diff, want, rtol=1e-9, atol=1e-9)


def pin_sampled_matches_full(o):
    """The one-at-a-time sampled outputs agree with the whole-matrix composites."""
    rng = np.random.default_rng(19)
    M, N, K, r = 7, 11, 256, 3
    x = _rand_x(rng, M, K)
    codes = rng.integers(0, 3, size=(N, K), dtype=np.uint8)
    sc = np.abs(rng.standard_normal((N, K // 128))).astype(np.float16).astype(np.float32)
    wq, d, _ = o.q2_pack(codes, sc)
    a, b = _rand_x(rng, r, K), _rand_x(rng, N, r)
    full = o.q2_lora_gemm(x, wq, d, a, b, N)
    mi = rng.integers(0, M, 20)
    ni = rng.integers(0, N, 20)
    got = o.q2_gemm_at(x, wq, d, N, mi, ni, a, b)
    assert np.allclose(got, full[mi, ni], rtol=1e-12, atol=1e-12)
    c4 = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    s = np.full((N, K // 64), 0.125, np.float32)
    z = np.full((N, K // 64), 7.5, np.float32)
    wq4, sz, _ = o.q4_pack(c4, s, z)
    full4 = o.q4_gemm(x, wq4, sz, N)
    assert np.allclose(o.q4_gemm_at(x, wq4, sz, N, mi, ni), full4[mi, ni], rtol=1e-12,
                       atol=1e-12)


def pin_q2_dual_is_the_split_concatenation(o):
    """A projection split along its input axis ("Slice weights, not activations"):
    x1 W1^T + x2 W2^T must equal the single product [x1 | x2] [W1 | W2]^T."""
    rng = np.random.default_rng(23)
    for M, N, K1, K2 in [(3, 5, 128, 384), (6, 4, 256, 256), (1, 9, 384, 128)]:
        x1, x2 = _rand_x(rng, M, K1), _rand_x(rng, M, K2)
        c1 = rng.integers(0, 3, size=(N, K1), dtype=np.uint8)
        c2 = rng.integers(0, 3, size=(N, K2), dtype=np.uint8)
        s1 = np.abs(rng.standard_normal((N, K1 // 128))).astype(np.float16).astype(np.float32)
        s2 = np.abs(rng.standard_normal((N, K2 // 128))).astype(np.float16).astype(np.float32)
        wq1, d1, _ = o.q2_pack(c1, s1)
        wq2, d2, _ = o.q2_pack(c2, s2)
        wq, d, _ = o.q2_pack(np.concatenate([c1, c2], axis=1), np.concatenate([s1, s2], axis=1))
        whole = o.q2_gemm(np.concatenate([x1, x2], axis=1), wq, d, N)
        dual = o.q2_dual_gemm(x1, wq1, d1, x2, wq2, d2, N)
        assert np.allclose(dual, whole, rtol=1e-12, atol=1e-12), (M, N, K1, K2)
        assert not np.allclose(dual, o.q2_gemm(x1, wq1, d1, N), rtol=1e-6, atol=1e-6)


def pin_q2_dual_closed_forms(o):
    """Second matrix all codes 1 (zero weights) or second activation zero: only the first
    product remains, exactly; and the sampled form matches the whole-matrix form."""
    rng = np.random.default_rng(29)
    M, N, K1, K2 = 4, 6, 256, 128
    x1, x2 = _rand_x(rng, M, K1), _rand_x(rng, M, K2)
    c1 = rng.integers(0, 3, size=(N, K1), dtype=np.uint8)
    s1 = np.full((N, K1 // 128), 0.5, np.float32)
    wq1, d1, _ = o.q2_pack(c1, s1)
    first = o.q2_gemm(x1, wq1, d1, N)
    wz, dz, _ = o.q2_pack(np.ones((N, K2), np.uint8), np.ones((N, K2 // 128), np.float32))
    assert np.array_equal(o.q2_dual_gemm(x1, wq1, d1, x2, wz, dz, N), first)
    c2 = rng.integers(0, 3, size=(N, K2), dtype=np.uint8)
    wq2, d2, _ = o.q2_pack(c2, np.full((N, K2 // 128), 0.25, np.float32))
    assert np.array_equal(o.q2_dual_gemm(x1, wq1, d1, np.zeros_like(x2), wq2, d2, N), first)
    full = o.q2_dual_gemm(x1, wq1, d1, x2, wq2, d2, N)
    mi, ni = rng.integers(0, M, 15), rng.integers(0, N, 15)
    assert np.allclose(o.q2_dual_gemm_at(x1, wq1, d1, x2, wq2, d2, N, mi, ni), full[mi, ni],
                       rtol=1e-12, atol=1e-12)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
