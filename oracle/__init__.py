"""fp64 CPU oracle for the Prism block-sparse video self-attention path.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA library and imports nothing from it.
"""
from .prism_oracle import *  # noqa: F401,F403
