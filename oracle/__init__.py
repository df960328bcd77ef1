"""CPU oracle for the SPA-Cache cached layer step and decode loop.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg may import this package.  It shares no code
with the CUDA library and never imports it; the product path does not fall
back to it.

See ``oracle/spa_oracle.py`` for the functions and the passages they follow.
"""
from .spa_oracle import *  # noqa: F401,F403
