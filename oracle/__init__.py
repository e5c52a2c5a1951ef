"""fp64 CPU oracle of the ViT encoder forward -- test infrastructure, not product code.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline leg and its
reference arm) may import this package.  The CUDA library never calls it and shares no code
with it.
"""
from .vit_oracle import *  # noqa: F401,F403
