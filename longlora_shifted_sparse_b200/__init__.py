"""B200-native S2-Attn (shifted sparse attention with RoPE + position interpolation).

The compute path is the C-ABI library ``libs2attn.so`` (hand-written sm_100a CUDA kernels);
``longlora_shifted_sparse_b200.s2attn`` is its thin ctypes binding. Importing the binding
fails loudly when the library has not been built.
"""
__all__ = ["flops"]
