"""Seeded synthetic workloads shared by the CUDA path's callers and the oracle.

Holds sizes and random draws only; none of the method's arithmetic lives here.
"""
from .configs import WORKLOADS, ORDER, Workload, get
from .gen import (Inputs, make_inputs, fastgen_policies, chunk_boundaries, decode_chunk_boundaries,
                  POL_TOPB, POL_MASS_COUNT, POL_LOCAL, POL_SPECIAL, POL_FULL, POL_CHUNK)

__all__ = ["WORKLOADS", "ORDER", "Workload", "get", "Inputs", "make_inputs",
           "fastgen_policies", "chunk_boundaries", "decode_chunk_boundaries", "POL_TOPB", "POL_MASS_COUNT",
           "POL_LOCAL", "POL_SPECIAL", "POL_FULL", "POL_CHUNK"]
