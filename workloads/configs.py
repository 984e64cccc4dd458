"""The five synthetic workloads of the decode hot path.

Each workload is one recurrent-layer shape (form, heads, d_k, d_v), a rank R and
a compression window W, a batch of requests, a dense prefill length and a number
of decode steps.  Value distributions are fixed per form in ``philox.py``.

Form orientation follows "Shallow Encoding Emits Deep Memories" (thelatestinai.com
figures & tables page), Table 17: for Mamba-2, d_k = d_B = 128 (the state
dimension) and d_v = d_x = 64 (the head dimension).
"""

from __future__ import annotations

import dataclasses
from dataclasses import dataclass

FORM_GDN = 0      # Gated DeltaNet: S <- g (I - b k k^T) S + b k v^T
FORM_KDA = 1      # Kimi Delta Attention: S <- (I - b k k^T) Diag(alpha) S + b k v^T
FORM_MAMBA2 = 2   # Mamba-2: S <- alpha S + Delta k v^T
FORM_NAMES = {FORM_GDN: "gdn", FORM_KDA: "kda", FORM_MAMBA2: "mamba2"}


@dataclass(frozen=True)
class Config:
    cid: int            # workload id, also the second Philox key word
    name: str
    form: int
    batch: int          # requests
    layers: int
    heads: int
    d_k: int
    d_v: int
    R: int
    W: int
    n_prefill: int      # dense prefill tokens before the conversion
    n_decode: int       # decode steps after the conversion
    vbar_unit: bool     # v̄ is a unit vector (else its norm is drawn from U(1, 4))
    seed: int = 0       # master seed, the first Philox key word

    @property
    def units(self) -> int:
        """Units (request, layer, head) in the whole workload."""
        return self.batch * self.layers * self.heads

    @property
    def units_per_layer(self) -> int:
        return self.batch * self.heads

    @property
    def m(self) -> int:
        """Factor columns just before a compression, R + W."""
        return self.R + self.W

    def replace(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)

    def unit_id(self, b: int, l: int, h: int) -> int:
        """Global unit index, request-major: ((b * layers) + l) * heads + h."""
        return (b * self.layers + l) * self.heads + h


CONFIGS = {
    # Tiny GDN check: 1 layer x 2 heads, 16x16, R=W=4, batch 1.
    0: Config(0, "tiny-gdn", FORM_GDN, batch=1, layers=1, heads=2, d_k=16, d_v=16,
              R=4, W=4, n_prefill=64, n_decode=32, vbar_unit=True),
    # One Qwen3.8-Flash-Next-shaped GDN layer, 48 heads of 128x128, batch 64.
    1: Config(1, "gdn-layer", FORM_GDN, batch=64, layers=1, heads=48, d_k=128, d_v=128,
              R=16, W=16, n_prefill=2048, n_decode=256, vbar_unit=False),
    # The full recurrent stack: 36 GDN layers x 48 heads, batch 256.
    2: Config(2, "gdn-stack", FORM_GDN, batch=256, layers=36, heads=48, d_k=128, d_v=128,
              R=16, W=16, n_prefill=4096, n_decode=1024, vbar_unit=False),
    # Mamba-2 form: 40 layers x 64 heads, d_state 128 x headdim 64, R=8, W=32.
    3: Config(3, "mamba2-stack", FORM_MAMBA2, batch=256, layers=40, heads=64, d_k=128, d_v=64,
              R=8, W=32, n_prefill=2048, n_decode=512, vbar_unit=False),
    # Kimi Delta Attention: 20 layers x 32 heads, 128x128, batch 512; R, W swept.
    4: Config(4, "kda-stack", FORM_KDA, batch=512, layers=20, heads=32, d_k=128, d_v=128,
              R=16, W=16, n_prefill=8192, n_decode=1024, vbar_unit=False),
}

KDA_SWEEP_R = (8, 16, 32)
KDA_SWEEP_W = (8, 16, 32, 64)


def config(cid: int, **overrides) -> Config:
    """A workload by id, optionally with fields replaced (smaller batch, fewer steps...)."""
    c = CONFIGS[cid]
    return c.replace(**overrides) if overrides else c
