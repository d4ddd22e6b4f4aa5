"""B200-native APB-V / Spava approximate-attention prefill (sm_100a).

The compute path is libspava.so (hand-written CUDA for sm_100a, C ABI in
include/spava.h); ``api`` wraps it for PyTorch tensors and streams, ``synth``
draws seeded video-shaped inputs.
"""
from .api import Layout, Spava, attended_pairs, packed_len, workspace_size  # noqa: F401
from .native import SpavaError  # noqa: F401
