"""Seeded synthetic inputs for the paged decode path.

This package is the one module both the GPU path and the oracle may use: it
draws sequence lengths, pool orders and stop decisions, and produces K/V/q
element values from a counter-based generator.  It contains none of the paging
or attention arithmetic.
"""
from . import values, workloads  # noqa: F401
