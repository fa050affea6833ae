"""Residual dual-scale binarized linear layer on NVIDIA B200 (sm_100a).

W ~= sum_{i=1..k} diag(g_i) B_i diag(h_i), B_i in {-1,+1}, derived as
B_i = sign(R_{i-1}) from the running residual (RaBiT, Algorithm 2 forward),
bit-packed, and applied as Y = sum_i g_i . (B_i (h_i . X)).

The compute lives in the C-ABI CUDA library ``librbw.so`` (see
``include/rbw.h``); ``residual_binarized_weight_b200.rbw`` is its thin ctypes
binding.  Importing this package does not load the library; the first call
into ``rbw`` does, and raises if it is missing.
"""
__all__ = ["rbw", "synth"]
