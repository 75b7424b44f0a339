"""B200-native (sm_100a) forward pass of Native Sparse Attention.

The compute path is the C-ABI library ``libnsa_b200.so`` (hand-written CUDA
for sm_100a, declared in ``include/nsa.h``); ``sparse_attention_long_06_b200.nsa``
is its thin ctypes binding over torch-allocated device memory and streams.
``workloads`` draws the seeded synthetic inputs.
"""
__all__ = ["nsa", "workloads"]
