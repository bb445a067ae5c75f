"""B200-native (sm_100a) block-sparse video self-attention forward.

The compute lives in ``libbsa.so`` (hand-written CUDA); this package is a
thin ctypes binding over its C ABI plus the seeded input generators.
"""
