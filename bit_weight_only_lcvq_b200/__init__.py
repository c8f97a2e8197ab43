"""liblcvq: B200-native LC-VQ 2-bit weight-only hot path.

``bit_weight_only_lcvq_b200.lcvq`` is the thin binding of the C ABI in
``include/lcvq.h``; ``bit_weight_only_lcvq_b200.synth`` holds the seeded
synthetic workloads.  Importing the package loads nothing: the library is
loaded on first use and every call fails loudly when it is missing.
"""
