"""B200 (sm_100a) implementation of the TurboQuant hot path.

The compute lives in the C-ABI CUDA library ``libtq.so`` (sources in ``csrc/``, declarations in
``include/tq.h`` at the repository root).  ``kv_cache_vector_06_b200.tq`` is the ctypes binding;
it raises on import if the library has not been built (``python -m kv_cache_vector_06_b200.build``).
"""
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtq.so")
