"""SeKV span-structured KV cache on B200 (sm_100a): C-ABI CUDA library + thin binding.

``sekv`` is the ctypes binding of ``include/sekv.h`` (same names as the C ABI);
``cache`` holds the torch-owned buffers the descriptors point at.
"""
from . import sekv
from .sekv import (SEKV_ATTEND, SEKV_BF16, SEKV_BUILD_ALL, SEKV_BUILD_BASES, SEKV_BUILD_LAYOUT,
                   SEKV_BUILD_SCAN, SEKV_BUILD_SUMMARY, SEKV_F32, SEKV_FUSED, SEKV_ROUTE, SekvError,
                   check)
from .cache import ColdFetcher, SpanCache, tau_to_theta

__all__ = ["sekv", "SpanCache", "ColdFetcher", "tau_to_theta", "SekvError", "check",
           "SEKV_FUSED", "SEKV_ROUTE", "SEKV_ATTEND", "SEKV_F32", "SEKV_BF16", "SEKV_BUILD_ALL",
           "SEKV_BUILD_SCAN", "SEKV_BUILD_LAYOUT", "SEKV_BUILD_SUMMARY", "SEKV_BUILD_BASES"]
