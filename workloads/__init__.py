"""Seeded synthetic workloads shared by the oracle side and the GPU side.

This package holds only input generation: the five workload definitions
(shapes, value distributions, lengths) and a host implementation of the
counter-based Philox4x32-10 generator (Salmon, Moraes, Dror, Shaw, "Parallel
random numbers: as easy as 1, 2, 3", SC'11) with the fixed transforms that turn
its words into q, k, v, alpha, beta and the per-head mean value v̄.

It contains none of the method's arithmetic (no recurrence, no factored update,
no compression).  The CUDA library carries its own, independently written
Philox generator for the same counters; the tests check that the two agree.
"""

from .configs import (CONFIGS, Config, FORM_GDN, FORM_KDA, FORM_MAMBA2, FORM_NAMES, KDA_SWEEP_R,
                      KDA_SWEEP_W, config)
from . import philox

__all__ = ["CONFIGS", "Config", "FORM_GDN", "FORM_KDA", "FORM_MAMBA2", "FORM_NAMES", "KDA_SWEEP_R",
           "KDA_SWEEP_W", "config", "philox"]
