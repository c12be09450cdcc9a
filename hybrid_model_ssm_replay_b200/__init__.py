"""Replay-based SSM decode for hybrid SSM/attention models on NVIDIA B200.

The compute path is librssm.so (hand-written sm_100a CUDA kernels behind the
C ABI of include/rssm.h); `rssm` is its thin ctypes binding and `inputs` the
seeded synthetic input recipe.
"""
