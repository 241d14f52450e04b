"""DS4 sparse-prefill attention on B200 (sm_100a).

The computation lives in libds4sp.so (csrc/, C ABI in include/ds4sp.h);
``ds4sp`` is its Python binding and ``inputs`` the seeded synthetic workloads.
Importing the package does not load the library; the first binding call does.
"""
from . import inputs  # noqa: F401
