"""Piecewise sparse attention (PISA) for NVIDIA B200 (sm_100a): C-ABI CUDA library + thin binding."""
