"""Exact softmax attention (causal / sliding-window / full GQA prefill and
paged decode) for NVIDIA B200, behind a C-ABI library of hand-written sm_100a
CUDA kernels. This module is the thin Python binding over that library."""
