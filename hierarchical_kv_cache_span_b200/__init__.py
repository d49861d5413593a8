"""SeKV span-structured KV cache on B200 (sm_100a): C-ABI CUDA library + thin binding.

``sekv`` is the ctypes binding of ``include/sekv.h`` (same names as the C ABI);
``cache`` holds the torch-owned buffers the descriptors point at. The library is
loaded on first use of any of these names (importing the package alone does not
load it, so ``python -m hierarchical_kv_cache_span_b200.build`` can rebuild it);
a missing library raises ImportError at that point - there is no fallback.
"""
import importlib

_FROM_SEKV = ("SEKV_ATTEND", "SEKV_BF16", "SEKV_BUILD_ALL", "SEKV_BUILD_BASES", "SEKV_BUILD_LAYOUT",
              "SEKV_BUILD_SCAN", "SEKV_BUILD_SUMMARY", "SEKV_F32", "SEKV_FUSED", "SEKV_ROUTE",
              "SekvError", "check")
_FROM_CACHE = ("ColdFetcher", "SpanCache", "tau_to_theta")

__all__ = ["sekv", "cache", *_FROM_SEKV, *_FROM_CACHE]


def __getattr__(name):
    if name in ("sekv", "cache"):
        return importlib.import_module(f".{name}", __name__)
    if name in _FROM_SEKV:
        return getattr(importlib.import_module(".sekv", __name__), name)
    if name in _FROM_CACHE:
        return getattr(importlib.import_module(".cache", __name__), name)
    raise AttributeError(name)
