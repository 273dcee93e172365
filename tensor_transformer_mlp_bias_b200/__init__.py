"""B200-native tensor-parallel Transformer MLP block with biases.

``inputs`` holds the seeded workload generators; ``binding`` is the thin
ctypes layer over the C-ABI library ``libmlptp.so`` built from ``csrc/``.
Importing the package does not load the CUDA library; the first call into
``binding`` does, and raises if it is missing.
"""
