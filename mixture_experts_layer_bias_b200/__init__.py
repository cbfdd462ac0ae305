"""B200-native (sm_100a) single-GPU Mixture-of-Experts layer forward.

The compute lives in the C-ABI shared library built from ``csrc/``
(libmoe_b200.so, declared in include/moe.h); ``ops`` is its thin ctypes
binding, ``layer`` a convenience owner of buffers.  Importing the package
does not load the library; the first call into ``ops`` does, and raises if
the library was not built.
"""

__all__ = ["ops", "synthetic"]
