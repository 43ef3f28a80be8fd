"""B200-native SPAttention band-sparse attention.

``head_partitioned_distance_b200.spa`` is the Python binding of the C-ABI
library ``libspa.so`` (hand-written sm_100a kernels); ``synth`` draws the
seeded synthetic inputs.  Importing this package loads nothing; importing
``spa`` loads the library and fails loudly when it has not been built.
"""
__all__ = ["spa", "synth"]
