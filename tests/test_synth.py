"""The seeded synthetic inputs follow their stated recipe (no GPU).

Each named workload has the stated shapes. Codes stay in their format's value set.
Scales and zeros are exact f16 values, as the packers require. The distributions match
their stated parameters within sampling error. The same seed gives the same input.
"""
import numpy as np
import pytest

from bit_weight_quantized_tgemm_b200 import synth


def _bf16_to_f32(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _is_f16_exact(a):
    return np.array_equal(a.astype(np.float16).astype(np.float32), a)


def test_named_workload_shapes():
    want = {
        "tiny": (16, 128, 256), "gemv_m1": (1, 3072, 3072), "gemv_m4": (4, 3072, 3072),
        "gemv_m16": (16, 3072, 3072), "mmdit_9216x3072": (1536, 9216, 3072),
        "mmdit_3072x12288": (1536, 3072, 12288), "mmdit_12288x3072": (1536, 12288, 3072),
        "lora_r4": (1536, 9216, 3072), "lora_r32": (1536, 9216, 3072),
        "lora_r64": (1536, 9216, 3072), "encoder_up": (512, 9728, 2560),
        "encoder_down": (512, 2560, 9728),
    }
    assert set(synth.ALL) == set(want)
    for name, (M, N, K) in want.items():
        w = synth.ALL[name]
        assert (w.M, w.N, w.K) == (M, N, K), name
    assert [synth.ALL[f"lora_r{r}"].r for r in (4, 32, 64)] == [4, 32, 64]
    assert synth.ALL["tiny"].out_f32 and not synth.ALL["mmdit_9216x3072"].out_f32


def test_flops_and_weight_bytes():
    w = synth.ALL["mmdit_9216x3072"]
    assert w.flops == 2 * 1536 * 9216 * 3072
    assert w.weight_bytes == 9216 * 3072 // 4 + 9216 * 24 * 2      # 2.125 bits a weight
    lo = synth.ALL["lora_r64"]
    assert lo.flops == 2 * 1536 * 9216 * 3072 + 2 * 1536 * 64 * (3072 + 9216)
    e = synth.ALL["encoder_up"]
    assert e.weight_bytes == 9728 * 2560 // 2 + 9728 * 40 * 4       # 4.5 bits a weight
    assert 8 * e.weight_bytes == 9728 * 2560 * 4.5


def test_ternary_recipe():
    p = synth.q2_problem(11, 64, 512, 1024, r=8)
    assert p.x.shape == (64, 1024) and p.x.dtype == np.uint16
    assert p.codes.shape == (512, 1024) and set(np.unique(p.codes)) == {0, 1, 2}
    assert p.scale.shape == (512, 8) and p.scale.dtype == np.float32
    assert _is_f16_exact(p.scale) and (p.scale >= 0).all()
    assert p.a.shape == (8, 1024) and p.b.shape == (512, 8)
    x = _bf16_to_f32(p.x)
    assert abs(x.mean()) < 0.02 and abs(x.std() - 1.0) < 0.02           # N(0, 1)
    # |N(0, 0.02)|: mean 0.02 * sqrt(2 / pi)
    assert abs(p.scale.mean() - 0.02 * np.sqrt(2 / np.pi)) < 0.002
    a = _bf16_to_f32(p.a)
    assert abs(a.std() - 1e-3) < 1e-4                                   # N(0, 1e-3)
    # uniform codes: each value about a third
    freq = np.bincount(p.codes.ravel(), minlength=3) / p.codes.size
    assert np.allclose(freq, 1 / 3, atol=0.01)


def test_gemv_code_mix():
    p = synth.ALL["gemv_m1"].make()
    freq = np.bincount(p.codes.ravel(), minlength=3) / p.codes.size
    assert np.allclose(freq, [0.3, 0.4, 0.3], atol=0.005)


def test_four_bit_recipe():
    p = synth.q4_problem(12, 32, 256, 640)
    assert p.codes.shape == (256, 640) and p.codes.max() <= 15
    assert len(np.unique(p.codes)) == 16
    assert p.s.shape == p.z.shape == (256, 10)
    assert _is_f16_exact(p.s) and _is_f16_exact(p.z)
    assert (p.z >= 7.0).all() and (p.z <= 8.0).all()                   # U[7, 8]
    assert abs(p.s.mean() - 0.01 * np.sqrt(2 / np.pi)) < 0.001          # |N(0, 0.01)|


def test_seeds_reproduce_and_differ():
    a = synth.q2_problem((5, 1), 8, 128, 256)
    b = synth.q2_problem((5, 1), 8, 128, 256)
    c = synth.q2_problem((5, 2), 8, 128, 256)
    assert np.array_equal(a.x, b.x) and np.array_equal(a.codes, b.codes)
    assert np.array_equal(a.scale, b.scale)
    assert not np.array_equal(a.codes, c.codes)


def test_block_size_rules():
    with pytest.raises(ValueError):
        synth.q2_problem(0, 1, 1, 192)
    with pytest.raises(ValueError):
        synth.q4_problem(0, 1, 1, 96)


def test_named_workload_seeds():
    # one seed per family: tiny 0, GEMV 1, MMDiT 2, branch 3, encoder 4
    want = {"tiny": 0, "gemv_m1": 1, "gemv_m4": 1, "gemv_m16": 1, "mmdit_9216x3072": 2,
            "mmdit_3072x12288": 2, "mmdit_12288x3072": 2, "lora_r4": 3, "lora_r32": 3,
            "lora_r64": 3, "encoder_up": 4, "encoder_down": 4}
    for name, seed in want.items():
        assert synth.ALL[name].seed == seed, name
    # the 1-token GEMV input is the first row of the 16-token one (same generator, same order)
    assert np.array_equal(synth.ALL["gemv_m1"].make().x[0], synth.ALL["gemv_m16"].make().x[0])
