"""B200 (sm_100a) ternary / 4-bit dequant-fused matmul library.

The compute lives in ``libtgemm.so`` (hand-written CUDA, C ABI in ``include/tgemm.h``);
this package is the Python binding (:mod:`.binding`) plus seeded synthetic workloads
(:mod:`.synth`).  PyTorch supplies device memory and streams only.
"""
from .binding import (  # noqa: F401
    DEVERR_TIMEOUT, EALIGN, EARCH, ECUDA, EINVAL, EWORKSPACE, OK, OP_Q2, OP_Q2_LORA, OP_Q4,
    OUT_BF16, OUT_F32, PACK_BAD_CODE, PACK_INEXACT, PACK_NONFINITE, PATH_AUTO, PATH_SMALL_M,
    PATH_SMALL_M_PASS, PATH_SMALL_M_STREAM, PATH_TENSOR, TgemmError, device_error, gemm_q2, gemm_q2_lora, gemm_q4, lib, library_path,
    q2_dequant, q2_pack, q4_dequant, q4_pack, set_path, version, workspace_size,
    workspace_size_min,
    KIND_GEMV_Q2, KIND_GEMV_Q4, KIND_PREP, KIND_TC_Q2, KIND_TC_Q2_LORA, KIND_TC_Q4,
    launch_count, profile_enable, profile_read, ETOOLARGE, NOALLOC_SCRATCH_BYTES,
    gemm_q2_noalloc, gemm_q2_dual, dual_workspace_size, tc_plan, TC_PLAN_KEYS,
    q2_from_gemlite, PACK_ZERO_MISMATCH, PACK_GROUP_MISMATCH, gemm_q2_lora_bt,
    selftest_wait_timeout, gemv_plan, GEMV_PLAN_KEYS, mma_rate,
)
