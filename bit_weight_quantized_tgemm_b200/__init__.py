"""B200 (sm_100a) ternary / 4-bit dequant-fused matmul library: Python binding."""
