"""The tensor-core schedule, checked on the host (no GPU needed).

tgemm_tc_plan reports the schedule the tensor-core kernel runs. This test restates the
kernel's index arithmetic in Python from the header's description: each CTA's two unit
ranges, its tile segments, the partial-sum slots, the arrival counters, the last arriver's
CTA range, and the dequant warps' incremental walk. It then checks, over many shapes and
SM counts, that:
- every (tile, stage) unit is run by exactly one CTA;
- each split tile's pieces come from consecutive CTAs, and each of those CTAs writes a
  slot that no other segment uses;
- counters stay inside the split region;
- the walk visits the units in the same order as the other roles;
- in the 4-bit all-split kernel, the CTAs that wait for later sharers at a tile's first
  k part wait only on higher-numbered CTAs that write their slots before any wait of
  their own, so the waits end.
A mistake in the host schedule, or a change to it that the kernel's index arithmetic
does not follow, fails here without a GPU.
"""
import random

import pytest

import bit_weight_quantized_tgemm_b200 as tg

pytestmark = pytest.mark.filterwarnings("ignore")


def _ranges(pl, c):
    ks = pl["ksteps"]
    units = pl["num_tiles"] * ks
    sk_u0 = pl["sk_t0"] * ks
    a0 = sk_u0 + c * pl["upc"]
    a1 = max(a0, min(units, a0 + pl["upc"]))
    b0 = c * pl["dpc"]
    b1 = max(b0, min(sk_u0, b0 + pl["dpc"]))
    return a0, a1, b0, b1


def _segments(pl, c):
    ks = pl["ksteps"]
    out = []
    for ua, ub in _ranges(pl, c)[:2], _ranges(pl, c)[2:]:
        u = ua
        while u < ub:
            t = u // ks
            end = min(ub, (t + 1) * ks)
            out.append((t, u - t * ks, end - t * ks))
            u = end
    return out


def _walk(pl, c):
    """The dequant warps' item-by-item advance (one compare per item)."""
    ks = pl["ksteps"]
    a0, a1, b0, b1 = _ranges(pl, c)
    n_first = a1 - a0
    n = n_first + (b1 - b0)
    in_first = n_first > 0
    u = a0 if in_first else b0
    tile, k = divmod(u, ks)
    seg_end = min(ks, a1 - tile * ks) if in_first else ks
    items = []
    for _ in range(n):
        items.append((tile, k))
        k += 1
        if k == seg_end:
            k = 0
            if in_first and tile * ks + seg_end == a1:
                in_first = False
                tile = b0 // ks
            else:
                tile += 1
            seg_end = min(ks, a1 - tile * ks) if in_first else ks
    return items


def check_plan(pl):
    ks, T = pl["ksteps"], pl["num_tiles"]
    assert pl["grid"] >= 1 and ks >= 1 and T >= 1
    if not pl["split"]:
        assert pl["sk_t0"] == 0 and pl["dpc"] == 0 and pl["upc"] % ks == 0
    else:
        assert pl["dpc"] % ks == 0 and 0 <= pl["sk_t0"] < T
    seen = {}
    slots = {}
    pieces = {}
    for c in range(pl["grid"]):
        segs = _segments(pl, c)
        flat = [(t, k) for t, ka, kb in segs for k in range(ka, kb)]
        assert flat == _walk(pl, c), f"dequant walk differs from the segments for CTA {c}"
        for it in flat:
            seen[it] = seen.get(it, 0) + 1
        for t, ka, kb in segs:
            if ka == 0 and kb == ks:
                continue  # a whole tile, stored straight from the accumulator
            t_rel = t - pl["sk_t0"]
            assert 0 <= t_rel < T - pl["sk_t0"], "a shared tile outside the split region"
            slot = 2 * c if c * pl["upc"] >= t_rel * ks else 2 * c + 1
            assert slot not in slots, f"slot {slot} written twice"
            assert slot < 2 * pl["grid"]
            slots[slot] = t
            pieces.setdefault(t, []).append(c)
    assert len(seen) == T * ks and set(seen.values()) == {1}, "units not covered exactly once"
    for t, cs in pieces.items():
        t_rel = t - pl["sk_t0"]
        lo, hi = t_rel * ks // pl["upc"], ((t_rel + 1) * ks - 1) // pl["upc"]
        assert sorted(cs) == list(range(lo, hi + 1)), f"tile {t}: pieces {cs}, expected {lo}..{hi}"


def _form(pl):
    if not pl["split"]:
        return "whole"
    return "hybrid" if pl["dpc"] > 0 else "split"


@pytest.mark.parametrize("op,M,N,K,r,K2,form", [
    (tg.OP_Q2, 1536, 9216, 3072, 0, 0, "whole"),     # 432 tiles = 3 x 144
    (tg.OP_Q2, 1536, 3072, 12288, 0, 0, "whole"),    # 144 tiles
    (tg.OP_Q4, 512, 9728, 2560, 0, 0, "split"),      # 152 tiles: 4 left over, cut over all CTAs
    (tg.OP_Q4, 512, 2560, 9728, 0, 0, "split"),      # 40 tiles
    (tg.OP_Q2, 1280, 9216, 3072, 0, 0, "hybrid"),    # 360 tiles: 2 waves + 64
    (tg.OP_Q2, 4096, 9216, 3072, 0, 0, "whole"),     # 1152 tiles: 7 waves + 116, split saves < its charge
    (tg.OP_Q2, 1536, 21504, 3072, 0, 0, "whole"),    # 1008 tiles: 6 waves + 120, likewise
    (tg.OP_Q2, 300, 13300, 3072, 0, 0, "hybrid"),    # 208 tiles: 1 wave + 60, ragged edges
    (tg.OP_Q2_LORA, 1280, 9216, 3072, 32, 0, "hybrid"),
    (tg.OP_Q2, 1536, 3072, 3072, 0, 12288, "whole"),  # fused out projection: 144 tiles of 120 stages
    (tg.OP_Q2, 256, 9216, 3072, 0, 0, "whole"),      # 72 tiles: halving K saves 12 units, less than the charge
    (tg.OP_Q2, 256, 1024, 4096, 0, 0, "split"),      # 8 tiles of 32 stages
])
def test_plan_forms(op, M, N, K, r, K2, form):
    pl = tg.tc_plan(op, M, N, K, r, K2, sms=148)
    assert _form(pl) == form, pl
    check_plan(pl)


def test_plan_invariants_random():
    rng = random.Random(20261202)
    forms = set()
    for _ in range(1500):
        op = rng.choice([tg.OP_Q2, tg.OP_Q2, tg.OP_Q4, tg.OP_Q2_LORA])
        M = rng.randint(1, 5000)
        N = rng.randint(1, 9000)
        K = 128 * rng.randint(1, 80)
        r = rng.choice([1, 4, 16, 17, 64, 256]) if op == tg.OP_Q2_LORA else 0
        K2 = 128 * rng.randint(1, 40) if op == tg.OP_Q2 and rng.random() < 0.2 else 0
        sms = rng.choice([148, 148, 148, 1, 2, 7, 100, 132, 160])
        pl = tg.tc_plan(op, M, N, K, r, K2, sms=sms)
        check_plan(pl)
        forms.add(_form(pl))
    assert forms == {"whole", "split", "hybrid"}


def test_plan_rejects_bad_arguments():
    for args in [(tg.OP_Q2, 0, 1, 128, 0, 0, 148), (tg.OP_Q2, 1, 1, 128, 0, 0, 0),
                 (7, 1, 1, 128, 0, 0, 148), (tg.OP_Q2_LORA, 1, 1, 128, 0, 0, 148),
                 (tg.OP_Q4, 1, 1, 128, 0, 128, 148)]:
        with pytest.raises(tg.TgemmError):
            tg.tc_plan(*args[:6], sms=args[6])


def test_plan_checker_catches_a_bad_schedule():
    """The checker itself rejects a plan whose ranges leave a unit out."""
    pl = tg.tc_plan(tg.OP_Q2, 1280, 9216, 3072, sms=148)
    bad = dict(pl, upc=pl["upc"] - 1)
    with pytest.raises(AssertionError):
        check_plan(bad)
