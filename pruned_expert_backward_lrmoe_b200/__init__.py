"""B200-native pruned MoE expert backward (LRMoE).

The compute path lives in the CUDA library ``liblrmoe.so`` built from ``csrc/``;
``lrmoe`` is its thin ctypes binding.  ``inputs`` draws seeded synthetic layers.
Importing this package does not load the CUDA library; the first call into
``lrmoe`` does, and raises if it is missing.
"""
