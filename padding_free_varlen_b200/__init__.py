"""Padding-free variable-length GPT-3 decoder-layer stack on B200 (sm_100a).

``capi``  - ctypes binding of the C-ABI library ``libenergon_rce.so``
            (offsets, transpose_padding_remove / rebuild, layer and stack forward).
``synth`` - the seeded synthetic-input generator shared with the tests.
``build`` - the in-tree nvcc build of the library.

Importing the package loads nothing; the CUDA library is loaded on the first
call through ``capi`` and a missing library is an error, never a fallback.
"""
