"""Seeded synthetic inputs for the SeKV span-cache hot path.

This package only draws random numbers and lays out tensors. It holds none
of the method's arithmetic: no boundary rule, no weights, no summaries, no
bases, no routing and no attention. The oracle (``oracle/``) and the CUDA
library (``hierarchical_kv_cache_span_b200``) both consume what it produces
and neither imports the other.
"""
from .gen import WORKLOADS, Workload, surprisal, keys_values, queries, taus, unit_seed

__all__ = ["WORKLOADS", "Workload", "surprisal", "keys_values", "queries", "taus", "unit_seed"]
