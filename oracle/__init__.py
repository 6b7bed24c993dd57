"""fp64 CPU oracle for the chunked TTT-KVB layer.

TEST INFRASTRUCTURE ONLY: imported by the test suite, by ``__graft_entry__.smoke()`` and
by the CPU-baseline legs of ``bench.py``. The C-ABI library and its Python binding never
import or execute anything here.
"""
from .ttt_oracle import *  # noqa: F401,F403
from . import ttt_oracle  # noqa: F401
