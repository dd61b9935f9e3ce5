"""B200-native per-token-group activation quantization.

The CUDA library (``libpqg.so``, built from ``csrc/``) is reached through the
C-ABI binding in ``precision_activation_quantization_b200.pqg``; importing that
module loads the library and fails loudly when it is missing.  ``inputs`` holds
the seeded synthetic workloads.
"""
