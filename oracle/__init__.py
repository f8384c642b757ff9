"""fp64 CPU oracle of the sharded-linear path.

TEST INFRASTRUCTURE ONLY: imported by the tests, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the product library.
"""
from .oracle import *  # noqa: F401,F403
from .oracle import OracleError, Partition, VocabLayout, LMHeadResult  # noqa: F401
