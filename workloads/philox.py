"""Host Philox4x32-10 and the fixed transforms that make the synthetic inputs.

Generator: Philox4x32-10 as defined by Salmon, Moraes, Dror and Shaw, "Parallel
random numbers: as easy as 1, 2, 3" (SC'11): a 4 x 32-bit counter, a 2 x 32-bit
key, ten rounds of two 32 x 32 -> 64-bit multiplies by 0xD2511F53 and
0xCD9E8D57 whose halves are xor-mixed with the other counter words and the key,
and a Weyl key schedule (+0x9E3779B9, +0xBB67AE85) between rounds.

Every value is addressed by its counter, so any subset of units and steps can be
regenerated independently on the host and on the device:

    key     = (master seed, workload id)
    counter = (block, field | phase << 8, t, unit)

``block`` indexes the group of four 32-bit words inside one field vector,
``field`` names the quantity (q, k, v, alpha, beta, v̄ ...), ``phase`` is 0 for
prefill tokens, 1 for decode steps and 2 for the lead-in steps of a request that
joined the batch earlier (ragged compression schedules), ``t`` is the token index
inside the phase, and ``unit`` is the global unit index ((b * L) + l) * H + h (per-head
quantities use l * H + h with t = 0).

Transforms, all evaluated in float64 and rounded to float32 once at the end:
  uniform  u = (x + 1/2) 2^-32 in (0, 1)
  normal   Box-Muller on consecutive word pairs: sqrt(-2 ln u0) (cos, sin)(2 pi u1)

Value distributions (the five workload definitions):
  GDN and KDA: k, q ~ N(0, I) then L2-normalised; v = 3 v̄ + 0.3 z; beta = sigmoid(z);
               GDN decay g = exp(-softplus(-3 + 0.5 z)); KDA alpha_i = 0.85 + 0.15 u_i.
  Mamba-2:     k, q ~ N(0, I) / sqrt(d_k); v = v̄ + 0.5 z; Delta = softplus(-2 + 0.5 z)
               (carried in the beta slot); alpha = exp(-Delta A) with A = 1 + 15 u per head.
  v̄:           a random direction, unit norm (tiny workload) or norm 1 + 3 u.
"""

from __future__ import annotations

import numpy as np

from .configs import Config, FORM_GDN, FORM_KDA, FORM_MAMBA2

_MASK = np.uint64(0xFFFFFFFF)
_M0 = np.uint64(0xD2511F53)
_M1 = np.uint64(0xCD9E8D57)
_W0 = np.uint64(0x9E3779B9)
_W1 = np.uint64(0xBB67AE85)
_SH = np.uint64(32)

# field ids (low byte of counter word 1)
F_Q, F_K, F_V, F_ALPHA, F_BETA = 0, 1, 2, 3, 4
F_VBAR_DIR, F_VBAR_NORM, F_A = 8, 9, 10
PHASE_PREFILL, PHASE_DECODE, PHASE_LEADIN = 0, 1, 2

_TWO_PI = 2.0 * np.pi
_U_SCALE = 2.0 ** -32


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Ten Philox4x32 rounds on broadcastable uint32-valued arrays; returns 4 word arrays."""
    c0, c1, c2, c3 = (np.asarray(x, dtype=np.uint64) for x in (c0, c1, c2, c3))
    k0 = np.asarray(k0, dtype=np.uint64)
    k1 = np.asarray(k1, dtype=np.uint64)
    for r in range(10):
        if r:
            k0 = (k0 + _W0) & _MASK
            k1 = (k1 + _W1) & _MASK
        p0 = c0 * _M0
        p1 = c2 * _M1
        c0, c1, c2, c3 = ((p1 >> _SH) ^ c1 ^ k0, p1 & _MASK, (p0 >> _SH) ^ c3 ^ k1, p0 & _MASK)
    return c0, c1, c2, c3


def _words(cfg: Config, unit, t, field: int, phase: int, n: int) -> np.ndarray:
    """The first n 32-bit words of one field vector, shape broadcast(unit, t) + (n,)."""
    nb = (n + 3) // 4
    unit = np.asarray(unit, dtype=np.uint64)[..., None]
    t = np.asarray(t, dtype=np.uint64)[..., None]
    blk = np.arange(nb, dtype=np.uint64)
    fw = np.uint64(field | (phase << 8))
    w = philox4x32_10(blk, fw, t, unit, np.uint64(cfg.seed), np.uint64(cfg.cid))
    shape = np.broadcast_shapes(unit.shape[:-1], t.shape[:-1]) + (nb,)
    out = np.stack([np.broadcast_to(x, shape) for x in w], axis=-1)  # (..., nb, 4)
    return out.reshape(shape[:-1] + (nb * 4,))[..., :n]


def uniforms(cfg: Config, unit, t, field: int, phase: int, n: int) -> np.ndarray:
    """n uniforms in (0, 1), float64."""
    return (_words(cfg, unit, t, field, phase, n).astype(np.float64) + 0.5) * _U_SCALE


def normals(cfg: Config, unit, t, field: int, phase: int, n: int) -> np.ndarray:
    """n standard normals by Box-Muller on word pairs (2i, 2i+1), float64."""
    n2 = n + (n & 1)
    u = uniforms(cfg, unit, t, field, phase, n2)
    r = np.sqrt(-2.0 * np.log(u[..., 0::2]))
    ang = _TWO_PI * u[..., 1::2]
    z = np.empty(u.shape, dtype=np.float64)
    z[..., 0::2] = r * np.cos(ang)
    z[..., 1::2] = r * np.sin(ang)
    return z[..., :n]


def _unit_norm(z: np.ndarray) -> np.ndarray:
    return z / np.sqrt(np.sum(z * z, axis=-1, keepdims=True))


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def _softplus(x):
    return np.log1p(np.exp(x))


def head_ids(cfg: Config, l, h):
    return np.asarray(l, dtype=np.int64) * cfg.heads + np.asarray(h, dtype=np.int64)


def vbar(cfg: Config, l, h) -> np.ndarray:
    """Per-head mean value v̄ for heads (l, h), float32, shape broadcast(l, h) + (d_v,)."""
    hid = head_ids(cfg, l, h)
    d = _unit_norm(normals(cfg, hid, 0, F_VBAR_DIR, PHASE_PREFILL, cfg.d_v))
    if cfg.vbar_unit:
        nrm = 1.0
    else:
        nrm = 1.0 + 3.0 * uniforms(cfg, hid, 0, F_VBAR_NORM, PHASE_PREFILL, 1)
    return (d * nrm).astype(np.float32)


def mamba2_A(cfg: Config, l, h) -> np.ndarray:
    """Mamba-2 per-head A ~ U(1, 16), float64, shape broadcast(l, h)."""
    hid = head_ids(cfg, l, h)
    return 1.0 + 15.0 * uniforms(cfg, hid, 0, F_A, PHASE_PREFILL, 1)[..., 0]


def vbar_table(cfg: Config) -> np.ndarray:
    """v̄ for every head, float32 [L][H][d_v]."""
    l, h = np.meshgrid(np.arange(cfg.layers), np.arange(cfg.heads), indexing="ij")
    return vbar(cfg, l, h)


def token_inputs(cfg: Config, b, l, h, t, phase: int, need_q: bool = True) -> dict:
    """Per-token inputs of units (b, l, h) at token t of ``phase`` (all broadcastable).

    Returns float32 arrays: q, k [..., d_k]; v [..., d_v]; alpha [...] (KDA: [..., d_k]);
    beta [...] (Mamba-2: Delta).
    """
    b, l, h, t = np.broadcast_arrays(*(np.asarray(x, dtype=np.int64) for x in (b, l, h, t)))
    unit = (b * cfg.layers + l) * cfg.heads + h
    vb = vbar(cfg, l, h).astype(np.float64)
    out = {}
    if cfg.form == FORM_MAMBA2:
        scale = 1.0 / np.sqrt(cfg.d_k)
        out["k"] = (normals(cfg, unit, t, F_K, phase, cfg.d_k) * scale).astype(np.float32)
        if need_q:
            out["q"] = (normals(cfg, unit, t, F_Q, phase, cfg.d_k) * scale).astype(np.float32)
        out["v"] = (vb + 0.5 * normals(cfg, unit, t, F_V, phase, cfg.d_v)).astype(np.float32)
        delta = _softplus(-2.0 + 0.5 * normals(cfg, unit, t, F_BETA, phase, 1)[..., 0])
        out["beta"] = delta.astype(np.float32)
        out["alpha"] = np.exp(-delta * mamba2_A(cfg, l, h)).astype(np.float32)
        return out
    out["k"] = _unit_norm(normals(cfg, unit, t, F_K, phase, cfg.d_k)).astype(np.float32)
    if need_q:
        out["q"] = _unit_norm(normals(cfg, unit, t, F_Q, phase, cfg.d_k)).astype(np.float32)
    out["v"] = (3.0 * vb + 0.3 * normals(cfg, unit, t, F_V, phase, cfg.d_v)).astype(np.float32)
    out["beta"] = _sigmoid(normals(cfg, unit, t, F_BETA, phase, 1)[..., 0]).astype(np.float32)
    if cfg.form == FORM_GDN:
        z = normals(cfg, unit, t, F_ALPHA, phase, 1)[..., 0]
        out["alpha"] = np.exp(-_softplus(-3.0 + 0.5 * z)).astype(np.float32)
    elif cfg.form == FORM_KDA:
        u = uniforms(cfg, unit, t, F_ALPHA, phase, cfg.d_k)
        out["alpha"] = (0.85 + 0.15 * u).astype(np.float32)
    else:
        raise ValueError(f"unknown form {cfg.form}")
    return out
