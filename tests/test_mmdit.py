"""The MMDiT step's linear inventory (host only).

The inventory is: 5 joint blocks of 4 linears per stream, 20 single blocks of a stacked
linear1 and a two-input linear2, and the text conditioning projection. These tests
check the counts, the shapes, the FLOP total, and that the row slices of linear1 tile its
packed matrix exactly.
"""
from bit_weight_quantized_tgemm_b200 import mmdit


def test_inventory_counts_and_shapes():
    seq = mmdit.step_linears(1024, 512)
    assert len(seq) == 1 + 5 * 2 * 4 + 20 * 2
    shapes = mmdit.weight_shapes()
    assert len(shapes) == 1 + 5 * 2 * 4 + 20 * 3
    for lin in seq:
        rows, k = shapes[lin.weight]
        assert k == lin.K and lin.row0 + lin.N <= rows
        if lin.K2:
            rows2, k2 = shapes[lin.weight2]
            assert k2 == lin.K2 and lin.row0 + lin.N <= rows2
    by_name = {lin.name: lin for lin in seq}
    assert (by_name["context"].M, by_name["context"].N, by_name["context"].K) == (512, 3072, 7680)
    assert (by_name["joint0.img.qkv"].M, by_name["joint0.txt.qkv"].M) == (1024, 512)
    l1, l2 = by_name["single0.linear1"], by_name["single0.linear2"]
    assert (l1.M, l1.N, l1.K) == (1536, 9216 + 12288, 3072)
    assert (l2.M, l2.N, l2.K, l2.K2) == (1536, 3072, 3072, 12288)


def test_flops_closed_form():
    img, txt = 1024, 512
    h, f = 3072, 12288
    joint = sum(2 * m * (3 * h * h + h * h + f * h + h * f) for m in (img, txt))
    single = 2 * (img + txt) * ((3 * h + f) * h + h * (h + f))
    total = 2 * txt * h * 7680 + 5 * joint + 20 * single
    assert sum(lin.flops for lin in mmdit.step_linears(img, txt)) == total


def test_row_slices_tile_linear1():
    whole = [l for l in mmdit.step_linears(slice_rows=False) if ".linear1" in l.name]
    parts = [l for l in mmdit.step_linears(slice_rows=True) if ".linear1" in l.name]
    assert len(parts) == 2 * len(whole)
    for w, (qkv, up) in zip(whole, zip(parts[0::2], parts[1::2])):
        assert qkv.weight == up.weight == w.weight
        assert (qkv.row0, qkv.N) == (0, 9216) and (up.row0, up.N) == (9216, 12288)
        assert qkv.N + up.N == w.N
    assert sum(l.flops for l in mmdit.step_linears(slice_rows=True)) == \
        sum(l.flops for l in mmdit.step_linears(slice_rows=False))
