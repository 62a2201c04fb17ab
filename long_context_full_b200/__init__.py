"""B200-native HySparse2 hybrid-block attention path.

``hs2``    - Python binding of the C ABI in include/hs2.h (libhs2.so, sm_100a)
``block``  - one Hybrid Block step (full attention + scores, selection, L
             sparse layers) built on that binding
``build``  - compiles libhs2.so in place with nvcc
"""
from . import hs2  # noqa: F401

__all__ = ["hs2"]
