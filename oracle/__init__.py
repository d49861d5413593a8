"""fp64 CPU oracle for SeKV's span-structured KV cache (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this package. The CUDA library never does, and this
package imports nothing from it.
"""
from .sekv_oracle import *  # noqa: F401,F403
from .sekv_oracle import __all__  # noqa: F401
