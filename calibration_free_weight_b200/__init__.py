"""HQQ zero-point solver for NVIDIA B200 (sm_100a): C-ABI library + thin binding."""
