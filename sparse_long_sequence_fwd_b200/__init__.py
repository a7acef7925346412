"""Longformer sparse self-attention forward for B200 (sm_100a).

The compute path is the C-ABI library ``liblfattn.so`` (hand-written CUDA);
``lf_attn`` is its thin ctypes binding.
"""
