"""Each planted mistake in the oracle must be caught by at least one pin (no GPU).

The mistakes are compiled into separate copies of the oracle (``ORACLE_PLANT_*``); the
real oracle is never modified.  A mistake that no pin catches would mean the pins do not
tie that part of the oracle to the pages.
"""
import pytest

from oracle import Oracle
from oracle_pins import ALL_PINS

PLANTS = [
    "ORACLE_PLANT_Q2_MSB_FIRST",      # wrong bit order
    "ORACLE_PLANT_Q2_NO_OFFSET",      # dropped the -1 in (q - 1) d
    "ORACLE_PLANT_Q2_SIGN",           # (1 - q) d
    "ORACLE_PLANT_Q2_SCALE_BLOCK64",  # scale indexed per 64 instead of per 128 weights
    "ORACLE_PLANT_Q4_NIBBLE_SWAP",    # even index in the high nibble
    "ORACLE_PLANT_Q4_ZERO_SIGN",      # (q + z) s
    "ORACLE_PLANT_F16_TRUNCATE",      # f32 -> f16 truncates instead of rounding
    "ORACLE_PLANT_GEMM_TRANSPOSED",   # transposed weight operand
    "ORACLE_PLANT_LORA_DROPPED",      # side branch missing
    "ORACLE_PLANT_DUAL_SECOND_DROPPED",  # split projection: second product missing
    "ORACLE_PLANT_GEMLITE_NO_TRANSPOSE",  # gemlite bytes read as [N][K/4]
    "ORACLE_PLANT_GEMLITE_ZERO_UNCHECKED",  # zeros == -scales not checked
    "ORACLE_PLANT_GEMLITE_GROUP_INDEX",  # block b takes group b mod (K/g)
    "ORACLE_PLANT_Q4_GROUP32",        # 4-bit group indexed per 32 instead of per 64 weights
    "ORACLE_PLANT_BF16_TRUNCATE",     # f64 -> bf16 output truncates instead of rounding
    "ORACLE_PLANT_LORA_A_TRANSPOSED",  # branch reads A as [K][r]
    "ORACLE_PLANT_LORA_B_TRANSPOSED",  # branch reads B as [r][N]
    "ORACLE_PLANT_SAMPLED_B_TRANSPOSED",  # sampled outputs alone read B as [r][N]
]


@pytest.mark.parametrize("plant", PLANTS)
def test_plant_is_caught(plant):
    mutant = Oracle(defines=(plant,))
    failed = []
    for pin in ALL_PINS:
        try:
            pin(mutant)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin catches {plant}"
