"""Seeded synthetic inputs shared by the tests, the oracle checks and the bench.

This package holds only random draws, shapes, lengths and page tables. It holds none of the
attention arithmetic: neither the oracle nor the CUDA path is imported here.
"""
from .inputs import *  # noqa: F401,F403
