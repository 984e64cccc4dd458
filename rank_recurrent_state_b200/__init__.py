"""SEED's sink-plus-low-rank recurrent state: the B200 decode hot path.

The compute lives in libseed.so (CUDA for sm_100a, C ABI in include/seed.h);
``rank_recurrent_state_b200.seed`` is the Python binding (torch for device memory
and streams).  Build the library with ``python -m rank_recurrent_state_b200.build``.
"""

__all__ = ["seed", "roofline"]
