"""CPU oracle (test infrastructure only) for the SmoothQuant W8A8 linear layer.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package; the product path never does.
"""
from .smoothquant import *  # noqa: F401,F403
from . import smoothquant  # noqa: F401
