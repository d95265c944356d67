"""B200-native Summaryformer frame memory and the attention that reads it.

The product is the C-ABI library ``libwmkv.so`` (``include/wmkv.h``): per-block
K/V buffers laid out | Z0 | RAW (Y+1) | SUM (W-Y) x X |, record writes,
RAW -> SUM eviction and a tcgen05 flash attention over the filled prefix, all
as hand-written sm_100a CUDA.  ``wmkv`` is its ctypes binding; it is loaded on
first use of any of its names (so that ``python -m
kv_memory_attention_b200.build`` can rebuild the library without loading it).
"""
import importlib


def __getattr__(name):
    if name.startswith("__"):
        raise AttributeError(name)
    if name == "build":
        # the build step must import without the library it builds
        return importlib.import_module(".build", __name__)
    mod = importlib.import_module(".wmkv", __name__)
    try:
        return getattr(mod, name)
    except AttributeError:
        raise AttributeError(f"module {__name__!r} has no attribute {name!r}") from None


def __dir__():
    mod = importlib.import_module(".wmkv", __name__)
    return sorted(set(globals()) | {n for n in vars(mod) if not n.startswith("_")})
