"""Seeded synthetic inputs for paged attention, shared by the CUDA path and the oracle.

This package holds no attention arithmetic: it only draws random numbers, rounds
them to the storage formats (bf16, fp8 e4m3) and lays out page tables.  Both the
GPU tests / benchmark and the float64 oracle consume exactly the bit patterns
produced here.
"""
from .gen import *  # noqa: F401,F403
