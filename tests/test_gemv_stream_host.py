"""The small-M streaming kernel's index arithmetic, restated and checked on the CPU (no GPU).

gemv_stream.cuh stages the activations of each 128-k unit in a permuted order and unpacks
each 32-bit word of packed codes into bf16 pairs with one lop3 per pair.  A and B of
mma.sync m16n8k16 must then agree on which k each slot holds.  This file restates, from
the kernel's description:
- the staging map (staged position 16 s + j of a unit holds k = stage_k(s, j));
- the pair extraction (mask a field, or in the exponent of the field's base);
- the fragment layouts of m16n8k16 (A: a0 (g, 2c..), a1 (g+8, 2c..), a2 (g, 2c+8..),
  a3 (g+8, 2c+8..); B: b0 (k 2c.., n g), b1 (k 2c+8.., n g); D: (g, 2c), (g, 2c+1),
  (g+8, 2c), (g+8, 2c+1)) and ldmatrix (lane (g, c) gets row g, columns 2c, 2c+1);
and checks that the emulated products, minus the correction sums the kernel forms, give
sum_k (q - 1) d x (Q2_0) and sum_k (q - z) s x (4-bit) for random codes and activations,
exactly (small integers).  It also checks the launch plan: the CTAs' row ranges and the
passes over K cover everything once, the swizzled code reads are conflict-free, and the
shared-memory layout fits and does not overlap.
"""
import itertools

import numpy as np
import pytest

import bit_weight_quantized_tgemm_b200 as tg


def stage_k(fmt, s, j):
    c, e, hi = (j & 7) >> 1, j & 1, j >> 3
    if fmt == 0:
        w, sp = c + 4 * (s >> 2), s & 3
        return 16 * w + 2 * sp + hi + 8 * e
    w, h = c + 4 * (s >> 1), s & 1
    return 8 * w + 2 * h + hi + 4 * e


def bf16_val(bits):
    return float(np.array([bits << 16], dtype=np.uint32).view(np.float32)[0])


def lop3_and_or(a, mask, orv):
    return ((a & mask) | orv) & 0xFFFFFFFF


def pair_vals(reg):
    return bf16_val(reg & 0xFFFF), bf16_val(reg >> 16)


def q2_pairs(w):
    w6, w12 = w >> 6, w >> 12
    return [lop3_and_or(w, 0x00030003, 0x43004300), lop3_and_or(w, 0x000C000C, 0x42004200),
            lop3_and_or(w, 0x00300030, 0x41004100), lop3_and_or(w6, 0x00030003, 0x43004300),
            lop3_and_or(w6, 0x000C000C, 0x42004200), lop3_and_or(w6, 0x00300030, 0x41004100),
            lop3_and_or(w12, 0x00030003, 0x43004300), lop3_and_or(w12, 0x000C000C, 0x42004200)]


def q4_pairs(w):
    return [lop3_and_or(w >> (4 * i), 0x000F000F, 0x43004300) for i in range(4)]


def q2_base(i):
    return (128, 32, 8)[(i & 7) % 3]


def test_stage_map_is_a_permutation():
    for fmt in (0, 1):
        ks = sorted(stage_k(fmt, s, j) for s in range(8) for j in range(16))
        assert ks == list(range(128)), fmt
        if fmt == 1:  # every k16 step lies in one 64-weight group
            for s in range(8):
                assert len({stage_k(1, s, j) // 64 for j in range(16)}) == 1


def test_pair_extraction_is_exact():
    rng = np.random.default_rng(0)
    for w in [int(v) for v in rng.integers(0, 2 ** 32, 200, dtype=np.uint64)]:
        codes = [(w >> (2 * i)) & 3 for i in range(16)]
        for i, reg in enumerate(q2_pairs(w)):
            lo, hi = pair_vals(reg)
            assert lo == q2_base(i) + codes[i] and hi == q2_base(i) + codes[i + 8]
        codes4 = [(w >> (4 * i)) & 15 for i in range(8)]
        for i, reg in enumerate(q4_pairs(w)):
            lo, hi = pair_vals(reg)
            assert lo == 128 + codes4[i] and hi == 128 + codes4[i + 4]


def _emulate_unit(fmt, words, xs):
    """One unit for 16 weight rows x 8 tokens: words[r][W] (row r's words), xs[m][k]
    (unit-relative k).  Returns per row/token the products of the kernel's operands,
    sum over the unit (Q2) or per group (4-bit), built fragment by fragment."""
    staged = np.zeros((8, 128))
    for m, s, j in itertools.product(range(8), range(8), range(16)):
        staged[m, 16 * s + j] = xs[m][stage_k(fmt, s, j)]
    ngroups = 1 if fmt == 0 else 2
    out = np.zeros((ngroups, 16, 8))
    for s in range(8):
        A = np.zeros((16, 16))
        B = np.zeros((16, 8))
        for g, c in itertools.product(range(8), range(4)):
            for r, rowbase in ((g, 0), (g + 8, 8)):
                if fmt == 0:
                    pr = q2_pairs(words[r][c + 4 * (s >> 2)])
                    lo_reg, hi_reg = pr[2 * (s & 3)], pr[2 * (s & 3) + 1]
                else:
                    pr = q4_pairs(words[r][c + 4 * (s >> 1)])
                    lo_reg, hi_reg = pr[2 * (s & 1)], pr[2 * (s & 1) + 1]
                A[r, 2 * c], A[r, 2 * c + 1] = pair_vals(lo_reg)       # a0 / a1
                A[r, 2 * c + 8], A[r, 2 * c + 9] = pair_vals(hi_reg)   # a2 / a3
            # ldmatrix: matrix 0 = staged [16 s, 16 s + 8), matrix 1 = [16 s + 8, 16 s + 16)
            B[2 * c, g], B[2 * c + 1, g] = staged[g, 16 * s + 2 * c], staged[g, 16 * s + 2 * c + 1]
            B[2 * c + 8, g] = staged[g, 16 * s + 8 + 2 * c]
            B[2 * c + 9, g] = staged[g, 16 * s + 9 + 2 * c]
        out[s // 4 if fmt == 1 else 0] += A @ B
    return out


@pytest.mark.parametrize("fmt", [0, 1])
def test_fragments_give_the_dequantized_product(fmt):
    rng = np.random.default_rng(1 + fmt)
    for _ in range(3):
        nw = 8 if fmt == 0 else 16
        words = [[int(v) for v in rng.integers(0, 2 ** 32, nw, dtype=np.uint64)] for _ in range(16)]
        xs = rng.integers(-4, 5, (8, 128)).astype(np.float64)
        prod = _emulate_unit(fmt, words, xs)
        if fmt == 0:
            codes = np.array([[(words[r][i // 16] >> (2 * (i % 16))) & 3 for i in range(128)]
                              for r in range(16)])
            corr = np.array([[sum((q2_base(k) + 1) * xs[m][k] for k in range(128)) for m in range(8)]])
            want = (codes - 1.0) @ xs.T
            assert np.array_equal(prod[0] - corr, want)
        else:
            codes = np.array([[(words[r][i // 8] >> (4 * (i % 8))) & 15 for i in range(128)]
                              for r in range(16)])
            z = rng.integers(0, 16, (16, 2)).astype(np.float64)
            for h in range(2):
                S = xs[:, 64 * h:64 * h + 64].sum(axis=1)
                got = prod[h] - (128.0 + z[:, h:h + 1]) * S[None, :]
                want = (codes[:, 64 * h:64 * h + 64] - z[:, h:h + 1]) @ xs[:, 64 * h:64 * h + 64].T
                assert np.array_equal(got, want)


SHAPES = [(0, 1, 3072, 3072), (0, 4, 3072, 3072), (0, 16, 3072, 3072), (0, 16, 21504, 3072),
          (0, 16, 3072, 12288), (0, 1, 12288, 3072), (1, 16, 9728, 2560), (1, 1, 2560, 9728),
          (1, 16, 2560, 9728), (1, 9, 2560, 9728), (0, 3, 136, 256), (1, 5, 100, 320),
          (0, 16, 1, 128), (1, 2, 7, 64), (0, 16, 520, 65536)]


@pytest.mark.parametrize("fmt,M,N,K", SHAPES)
@pytest.mark.parametrize("sms", [148, 132, 7])
def test_plan_covers_rows_and_k_once(fmt, M, N, K, sms):
    pl = tg.gemv_plan(fmt, M, N, K, sms)
    if pl is None:
        # no layout fits (on very few SMs a CTA's rows carry too many scales to stage):
        # the per-pass kernel serves the call; never on a full B200
        assert sms < 100, (fmt, M, N, K, sms)
        return
    assert pl["T"] == (1 if M <= 8 else 2)
    assert pl["grid"] == sms or (pl["T"] == 1 and pl["grid"] == 2 * sms and pl["smem"] <= 115712
                                 and pl["passes"] == -(-((K + 127) // 128) // 32))
    assert 2 <= pl["S"] <= 4
    U = (K + 127) // 128
    assert pl["U"] == U
    # passes: kp a multiple of 128 (whole units), at most 4096; the passes cover K once
    kp, P = pl["kp"], pl["passes"]
    assert kp % 128 == 0 and kp <= 4096 and P == -(-U // (kp // 128))
    assert (P - 1) * kp < 128 * U <= P * kp
    # row ranges: 8-row aligned, contiguous, covering [0, N), at most j_max tiles of 32
    n8 = (N + 7) // 8
    grid = pl["grid"]
    rows = [(8 * (c * n8 // grid), min(N, 8 * ((c + 1) * n8 // grid))) for c in range(grid)]
    assert rows[0][0] == 0 and rows[-1][1] == N
    for (a0, a1), (b0, _) in zip(rows, rows[1:]):
        assert a1 == b0 or (a1 == N and b0 >= N)
    assert max(-(-max(b - a, 0) // 32) for a, b in rows) <= pl["j_max"]
    # shared memory: regions in order, aligned, inside the budget
    T = pl["T"]
    offs = [pl["off_x"], pl["off_corr"], pl["off_red"], pl["off_acc"], pl["off_sc"], pl["off_ring"],
            pl["off_bar"]]
    assert offs == sorted(offs) and pl["off_ring"] % 1024 == 0 and pl["off_bar"] % 8 == 0
    assert pl["off_corr"] >= M * pl["xs_stride"] and pl["xs_stride"] >= 2 * kp
    assert pl["off_red"] - pl["off_corr"] >= (kp // 128) * (1 if fmt == 0 else 2) * 16 * 4
    assert pl["off_acc"] - pl["off_red"] >= 2 * 8 * 32 * 8 * T * 4
    if P > 1:
        assert pl["off_sc"] - pl["off_acc"] >= pl["j_max"] * 32 * 8 * T * 4
    assert pl["off_ring"] - pl["off_sc"] >= pl["j_max"] * 32 * U * (2 if fmt == 0 else 8)
    code_bytes = kp // 4 if fmt == 0 else kp // 2
    assert pl["nbox"] == -(-code_bytes // 128)
    assert pl["off_ring"] + pl["S"] * pl["nbox"] * 32 * 128 <= pl["off_bar"]
    assert pl["smem"] <= 232448 and pl["smem"] >= pl["off_bar"] + 2 * pl["S"] * 8 + 8 + 1024
    assert pl["xs_stride"] % 128 == 16
    # TMA boxes: every box's x coordinate is a multiple of 16 bytes
    row_bytes = K // 4 if fmt == 0 else K // 2
    assert row_bytes % 16 == 0
    for p_ in range(P):
        assert all((p_ * code_bytes + 128 * b) % 16 == 0 for b in range(pl["nbox"]))


def code_addr(r, w):
    """Byte offset of 32-bit word w of row r in a slot of 128-byte-swizzled 32 x 128 boxes."""
    b, o = w >> 5, (w & 31) * 4
    return b * 4096 + r * 128 + ((((o >> 4) ^ (r & 7)) << 4) | (o & 15))


def test_swizzled_code_reads_are_conflict_free_and_in_place():
    # the 128-byte swizzle moves 16-byte chunk i of row r to chunk i ^ (r % 8)
    for r in range(32):
        for w in range(64):
            a = code_addr(r, w)
            b, o = w >> 5, (w & 31) * 4
            assert a // 4096 == b and (a % 4096) // 128 == r
            assert ((a % 128) >> 4) == ((o >> 4) ^ (r & 7)) and a % 16 == o % 16
    # one warp's word reads (lane (g, c): row g + 8 r, words uw + c + 4 hw (Q2) or uw + word
    # (4-bit)) touch 32 distinct banks
    for fmt in (0, 1):
        for u in range(8):
            uw = u * (8 if fmt == 0 else 16)
            for half, r in itertools.product(range(2 if fmt == 0 else 4), range(4)):
                addrs = []
                for g in range(8):
                    for c in range(4):
                        w = uw + c + 4 * half
                        addrs.append(code_addr(g + 8 * r, w))
                banks = {}
                for a in addrs:
                    banks.setdefault((a // 4) % 32, set()).add(a)
                assert all(len(v) == 1 for v in banks.values()), (fmt, u, half)
