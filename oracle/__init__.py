"""CPU float64 oracle of MLA absorbed decode -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package. It never imports the CUDA library and the library never imports it.
"""
from . import compare, kv_accounting, mla_ref  # noqa: F401
