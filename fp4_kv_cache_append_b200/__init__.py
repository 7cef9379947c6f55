"""B200-native CSA2 sparse attention over an FP4 KV cache.

The compute path is the C-ABI library ``libcsa2.so`` (hand-written sm_100a
CUDA kernels, see ``include/csa2.h``); :mod:`.csa2` is its thin ctypes binding.
:mod:`.inputs` holds the seeded synthetic workloads.  Importing the package
does not load the library; the first call through :mod:`.csa2` does, and
fails loudly when it is missing.
"""
__all__ = ["csa2", "inputs"]
