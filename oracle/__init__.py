"""fp64 CPU oracle for ACE expert skipping -- test infrastructure only.

Imported by ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py``; never by the product package.  Nothing here is a fallback.
"""
from .oracle import *  # noqa: F401,F403
from .oracle import lib, set_threads, threads  # noqa: F401
