"""Padding-free variable-length GPT-3 decoder-layer stack on B200 (sm_100a).

The CUDA library and its Python binding are added in ``capi``.
"""
