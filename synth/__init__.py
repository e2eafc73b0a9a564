"""Seeded synthetic inputs for SageSLA attention.

This package only draws random numbers and stores them as bf16 bit patterns.
It holds none of the attention method's arithmetic, so both the CPU oracle and
the CUDA path can consume the very same bytes.
"""

from .workloads import CONFIGS, SWEEP_FRACS, Workload, make_inputs, make_workload, nblk_of

__all__ = ["CONFIGS", "SWEEP_FRACS", "Workload", "make_inputs", "make_workload", "nblk_of"]
