"""fp64 CPU oracle for exact attention.  Test infrastructure only: imported by
``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``,
never by the CUDA library or its Python binding."""

from .attention import *  # noqa: F401,F403
from .attention import __all__  # noqa: F401
