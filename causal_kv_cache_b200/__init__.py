"""causal_kv_cache_b200 -- the Ca2-VDM cached attention path on one NVIDIA B200 (sm_100a).

The compute lives in ``libca2.so`` (CUDA kernels behind the C ABI of ``include/ca2.h``);
``ca2`` is the ctypes binding with the same function names.  There is no CPU fallback:
importing the binding fails loudly when the library has not been built.
"""
from .ca2 import *  # noqa: F401,F403
from .ca2 import __all__  # noqa: F401
