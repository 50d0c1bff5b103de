"""B200-native Spherical KV: Angle-Domain Attention paged decode.

The CUDA kernels and the C-ABI live in ``csrc/`` and build into
``libskv.so`` next to this file; ``skv`` is the thin ctypes binding over it.
Importing the package does not load the library; ``skv.lib()`` does.
"""
