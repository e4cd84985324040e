"""Seeded synthetic inputs for the In-Place TTT fast-weight MLP layer.

This package holds the workload definitions and the seeded input generator
shared by the CUDA path's tests/benchmark and by the CPU oracle.  It contains
none of the layer's arithmetic: only random draws, the RMS normalisation of
the input rows that the workload recipe asks for, and rounding to the
storage precision.
"""

from .inputs import WORKLOADS, Workload, make_inputs, round_to_bf16, small_case, workload

__all__ = ["WORKLOADS", "Workload", "make_inputs", "round_to_bf16", "small_case", "workload"]
