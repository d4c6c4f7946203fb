"""fp64 CPU oracle for the LIME hot path — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The CUDA library and its Python binding never
import it, and the two share no code.
"""
from .lime_oracle import *  # noqa: F401,F403
