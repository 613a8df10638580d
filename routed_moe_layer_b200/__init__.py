"""B200 (sm_100a) routed MoE block: fp32 group-limited sigmoid router,
token permutation and tcgen05 grouped SwiGLU experts behind a C-ABI library.

The compute path lives in ``libroutedmoe.so`` (``csrc/``); ``ops`` is a thin
ctypes binding over it.  Importing the package does not load the library;
the first call into ``ops`` does, and fails loudly when it is missing.
"""

__all__ = ["inputs", "ops"]
