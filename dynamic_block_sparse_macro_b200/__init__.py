"""B200-native (sm_100a) Prism dynamic block-sparse video self-attention.

The compute path is the CUDA library ``libprism.so`` (C ABI in
``include/prism.h``); this package holds its ctypes binding (``_abi``), a
layer object that owns device buffers and issues the ABI calls in order
(``layer``), the workload table (``configs``) and the seeded synthetic input
generators (``inputs``).  Importing the package does not load the library;
the first ABI call does, and fails loudly if it has not been built.
"""

__all__ = ["configs", "inputs"]


def __getattr__(name):
    if name in ("PrismSparseAttention", "prism_attention"):
        from . import layer
        return getattr(layer, name)
    raise AttributeError(name)
