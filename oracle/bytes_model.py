"""Analytical byte account of one request's recurrent state (oracle).

SEED figures & tables (thelatestinai.com), Table 17 ("Analytical byte and FLOP
account"):
  dense state per head   b_s d_k d_v
  shallow state per head b_s [d_k + (d_k + d_v)(R + w)] at w steps after a
                         compression, 0 <= w <= W (the sink's coefficient and the
                         factors; the shared mean direction v̄ is not counted)
  resident request       state bytes + T x attention-cache bytes per token
                         (short-convolution windows left out, as in Table 2)
Table 2 on the same page reports these per request in MB = 10^6 bytes, at
w = 0 ("at R"), w = W/2 ("mean, R+W/2") and w = W ("peak, R+W").
"""

from __future__ import annotations


def dense_state_bytes(heads: int, d_k: int, d_v: int, b_s: int = 4) -> int:
    """Dense recurrent state of ``heads`` heads: heads * b_s * d_k * d_v."""
    return heads * b_s * d_k * d_v


def shallow_state_bytes(heads: int, d_k: int, d_v: int, R: int, w: int, b_s: int = 4) -> int:
    """Sink coefficient plus factors at w steps after a compression."""
    return heads * b_s * (d_k + (d_k + d_v) * (R + w))


def resident_bytes(state_bytes: float, tokens: int, cache_bytes_per_token: int) -> float:
    """State bytes plus the attention cache of ``tokens`` tokens."""
    return state_bytes + tokens * cache_bytes_per_token
