"""B200-native Geometric Context Attention (GCA) hot path.

``gca``    — ctypes binding of the C-ABI library ``libgca.so`` (built from
             ``csrc/`` for sm_100a); loading it fails loudly when it is missing.
``inputs`` — seeded synthetic streams of the five workloads.
The binding is imported lazily so that ``inputs`` works without the library.
"""
__all__ = ["gca", "inputs"]
