"""fp64 CPU oracle of the Veda block-sparse attention path -- test infrastructure.

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import this package. The CUDA library never does, and this package never imports it.
"""
from .veda_oracle import *  # noqa: F401,F403
from . import veda_oracle  # noqa: F401
