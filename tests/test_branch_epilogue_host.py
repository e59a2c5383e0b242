"""Index arithmetic of two pieces of the matmul kernels, restated and checked on the CPU.

1. The small-M branch's u = x A^T (lora_down_small_kernel): lane (g, c) of a warp feeds
   the k slots {2c, 2c+1, 2c+8, 2c+9} of an mma.sync m16n8k16 step with elements
   4c .. 4c+3 of that step (one 8-byte load per row), for both operands: A (16 token rows
   of x) and B (8 rows of A).  Emulating the m16n8k16 fragment layouts (A: a0 (g, 2c..),
   a1 (g+8, 2c..), a2 (g, 2c+8..), a3 (g+8, 2c+8..); B: b0 (k 2c.., n g), b1 (k 2c+8..,
   n g); D: (g, 2c), (g, 2c+1), (g+8, 2c), (g+8, 2c+1)) over every step must give
   x A^T exactly (small integers), and the per-warp sums added in warp order must cover
   every step once.
2. The tensor-core kernel's bf16 output of a whole tile: warp (q, eh) of the epilogue holds
   weight rows 32 q .. 32 q + 31 (one per lane) for the tokens of column half eh; each
   32-token chunk goes to a [32 tokens][128 rows] box (element (token e, row 32 q + lane)),
   then warp q writes token rows 8 q .. 8 q + 7 of the chunk, lane l covering rows
   4 l .. 4 l + 3, to y.  Every (token, row) of the tile must be written exactly once,
   with its own value, and nothing past M or N.
"""
import numpy as np
import pytest


def mma_m16n8k16(a_frag, b_frag):
    """D (16 x 8) of one m16n8k16 step from per-lane fragments a_frag[lane] = (a0, a1, a2, a3),
    each a pair (lo, hi) of values, and b_frag[lane] = (b0, b1)."""
    A = np.zeros((16, 16))
    B = np.zeros((16, 8))
    for lane in range(32):
        g, c = lane >> 2, lane & 3
        a0, a1, a2, a3 = a_frag[lane]
        A[g, 2 * c:2 * c + 2] = a0
        A[g + 8, 2 * c:2 * c + 2] = a1
        A[g, 2 * c + 8:2 * c + 10] = a2
        A[g + 8, 2 * c + 8:2 * c + 10] = a3
        b0, b1 = b_frag[lane]
        B[2 * c:2 * c + 2, g] = b0
        B[2 * c + 8:2 * c + 10, g] = b1
    return A @ B


@pytest.mark.parametrize("M,K,r", [(16, 256, 8), (5, 384, 3), (12, 3072, 8)])
def test_lora_down_small_fragment_map(M, K, r):
    rng = np.random.default_rng(7 + M + K + r)
    x = rng.integers(-3, 4, size=(M, K)).astype(np.float64)
    a = rng.integers(-3, 4, size=(r, K)).astype(np.float64)
    warps = 16
    steps = K // 16
    red = np.zeros((warps, 16, 8))
    seen = np.zeros(steps, dtype=int)
    for w in range(warps):
        acc = np.zeros((16, 8))
        for kb in range(w, steps, warps):  # interleaved k16 steps
            seen[kb] += 1
            a_frag, b_frag = [], []
            for lane in range(32):
                g, c = lane >> 2, lane & 3
                e0 = 16 * kb + 4 * c  # this lane's 4 elements of the step
                row0 = x[g, e0:e0 + 4] if g < M else np.zeros(4)
                row1 = x[g + 8, e0:e0 + 4] if g + 8 < M else np.zeros(4)
                arow = a[g, e0:e0 + 4] if g < r else np.zeros(4)
                # f0 = (x0, y0), f1 = (x1, y1) as uint2: af = {f0.x, f1.x, f0.y, f1.y}
                a_frag.append((row0[0:2], row1[0:2], row0[2:4], row1[2:4]))
                b_frag.append((arow[0:2], arow[2:4]))
            acc += mma_m16n8k16(a_frag, b_frag)
        red[w] = acc
    assert (seen == 1).all(), "every k16 step runs exactly once"
    u = red.sum(axis=0)  # the kernel adds the warps in order; integers, so order is immaterial
    ref = x @ a.T
    np.testing.assert_array_equal(u[:M, :r], ref)
    assert not u[M:, :].any() and not u[:, r:].any()


@pytest.mark.parametrize("M,N,tm,tn", [(256, 256, 0, 1), (300, 300, 1, 2), (40, 132, 0, 1)])
def test_whole_tile_output_boxes(M, N, tm, tn):
    """One 128-row x 256-token tile (token block tm, row block tn) through the boxes."""
    rng = np.random.default_rng(11)
    acc = rng.standard_normal((128, 256))  # accumulator: [row][token] of the tile
    y = np.full((M, N), np.nan)
    writes = np.zeros((M, N), dtype=int)
    for eh in range(2):  # column half of the accumulator
        mbase = tm * 256 + eh * 128
        for cc in range(4):  # 32-token chunks
            box = np.full((32, 128), np.nan)
            for q in range(4):
                for lane in range(32):
                    for e in range(32):
                        box[e, q * 32 + lane] = acc[q * 32 + lane, eh * 128 + cc * 32 + e]
            assert not np.isnan(box).any(), "the 4 warps fill the whole box"
            for q in range(4):
                m0 = mbase + cc * 32 + 8 * q
                for lane in range(32):
                    n4 = tn * 128 + 4 * lane
                    rows = min(8, M - m0) if n4 < N else 0
                    for e8 in range(8):
                        if e8 < rows:
                            for j in range(4):  # the 8-byte store covers rows n4 .. n4 + 3
                                assert n4 + j < N, "N % 4 == 0 keeps a store inside the row"
                                y[m0 + e8, n4 + j] = box[8 * q + e8, 4 * lane + j]
                                writes[m0 + e8, n4 + j] += 1
    m_lo, m_hi = tm * 256, min(M, tm * 256 + 256)
    n_lo, n_hi = tn * 128, min(N, tn * 128 + 128)
    assert (writes[m_lo:m_hi, n_lo:n_hi] == 1).all(), "every (token, row) of the tile once"
    assert writes.sum() == (m_hi - m_lo) * (n_hi - n_lo), "nothing outside the tile or past M, N"
    np.testing.assert_array_equal(y[m_lo:m_hi, n_lo:n_hi], acc[:n_hi - n_lo, :m_hi - m_lo].T)
