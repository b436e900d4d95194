"""MXFP8 quantisation and dropless grouped GEMM for B200 (sm_100a)."""
