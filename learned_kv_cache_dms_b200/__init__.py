"""B200-native Dynamic Memory Sparsification (DMS) inference hot path.

The compute path lives in the CUDA library ``libdms.so`` (C ABI declared in
``include/dms.h``); ``learned_kv_cache_dms_b200.binding`` is its thin Python
binding.  Importing this package does not load the library; importing the
binding does, and fails loudly if it has not been built.
"""
__version__ = "0.1.0"
