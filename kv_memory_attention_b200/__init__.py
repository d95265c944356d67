"""B200-native Summaryformer frame memory and the attention that reads it.

The product is the C-ABI library ``libwmkv.so`` (``include/wmkv.h``): per-block
K/V buffers laid out | Z0 | RAW (Y+1) | SUM (W-Y) x X |, record writes,
RAW -> SUM eviction and a tcgen05 flash attention over the filled prefix, all
as hand-written sm_100a CUDA.  ``wmkv`` is its ctypes binding.
"""
from .wmkv import *  # noqa: F401,F403
from .wmkv import KVMemory, WmError, LIB, LIB_PATH, SIGNATURES  # noqa: F401
