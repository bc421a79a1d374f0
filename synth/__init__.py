"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the oracle.

This package holds no arithmetic of the method: it draws random values, context
lengths and free-list orders, and drives whatever block allocator it is handed
(``bm``: an object with ``allocate(n)``, ``share(ids)``, ``copy_on_write(id)``) to lay
sequences out in the pool.  Slot mappings, quantisation, gathering and attention are
computed by the code under test (the CUDA library) or by the oracle, never here.
"""
from .workloads import PRESETS, Workload, build_workload  # noqa: F401
