"""Seeded synthetic inputs and the workload shapes of the sharded-linear path.

Shared by the tests, the bench and the oracle harness; holds none of the
method's arithmetic.
"""
from . import gen, configs  # noqa: F401
