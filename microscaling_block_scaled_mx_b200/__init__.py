"""MX (microscaling) cast and block-scaled GEMM for NVIDIA B200 (sm_100a)."""
