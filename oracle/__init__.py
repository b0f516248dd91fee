"""CPU oracle for the SparsePR attention call -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its
``cpu_baseline`` leg and ``--impl reference`` arm) may import this package. The
product path (the CUDA library and its Python binding) never imports, calls or
links anything here, and this package imports nothing from the product.
"""
from .sparsepr import *  # noqa: F401,F403
from .sparsepr import __all__  # noqa: F401
