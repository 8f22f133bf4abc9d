"""B200-native (sm_100a) exact attention: forward / backward behind a C ABI (libfa.so).

Import ``exact_io_aware_88_b200.fa`` for the binding; it loads the in-tree libfa.so and
fails loudly if it is absent.
"""
__all__ = ["fa"]
