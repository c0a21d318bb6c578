"""Seeded synthetic inputs, shared by the CPU oracle and the CUDA path.

Holds only random-number generation and workload shapes; no step of the
Medusa method is computed here.
"""
from . import gen, synth, workloads  # noqa: F401
