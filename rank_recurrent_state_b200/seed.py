"""Python binding of libseed.so: argument marshalling only.

Every function here has the name of the C entry point it calls (include/seed.h,
include/seed_synth.h), takes torch tensors for the device pointers, passes
``tensor.data_ptr()`` and the current CUDA stream, and raises ``SeedError`` on a
negative status.  All arithmetic happens in the library's kernels; torch only
provides device memory and streams.
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib

SEED_GDN, SEED_KDA, SEED_MAMBA2 = 0, 1, 2
SEED_ALL_LAYERS = -1
SEED_PHASE_PREFILL, SEED_PHASE_DECODE, SEED_PHASE_LEADIN = 0, 1, 2
SEED_MAX_COLS = 96
SEED_FACTORS_F32, SEED_FACTORS_F16, SEED_FACTORS_BF16 = 0, 1, 2
FACTOR_DTYPES = {SEED_FACTORS_F32: torch.float32, SEED_FACTORS_F16: torch.float16,
                 SEED_FACTORS_BF16: torch.bfloat16}
FACTOR_NAMES = {"f32": SEED_FACTORS_F32, "f16": SEED_FACTORS_F16, "bf16": SEED_FACTORS_BF16}

FLAG_FULL = 0x1
FLAG_NONFINITE = 0x2
FLAG_NOCONVERGE = 0x4
FLAG_BADCOLS = 0x8
FLAG_ZERO_VBAR = 0x10
FLAG_BADINDEX = 0x20
FLAG_TIMEOUT = 0x40


class SeedError(RuntimeError):
    def __init__(self, fn: str, status: int):
        lib = _lib.load()
        msg = lib.seed_status_string(status).decode()
        super().__init__(f"{fn} returned {status} ({msg})")
        self.status = status


@dataclass(frozen=True)
class Dims:
    form: int
    batch: int
    layers: int
    heads: int
    d_k: int
    d_v: int
    R: int
    W: int
    factors: int = SEED_FACTORS_F32   # element type of U and V

    @property
    def m(self) -> int:
        return self.R + self.W

    @property
    def units(self) -> int:
        return self.batch * self.layers * self.heads

    def c(self) -> _lib.seed_dims:
        return _lib.seed_dims(self.form, self.batch, self.layers, self.heads, self.d_k, self.d_v,
                              self.R, self.W, self.factors)

    @property
    def factor_dtype(self) -> torch.dtype:
        return FACTOR_DTYPES[self.factors]

    @staticmethod
    def from_config(cfg, batch: int | None = None, factors: int = SEED_FACTORS_F32) -> "Dims":
        return Dims(cfg.form, cfg.batch if batch is None else batch, cfg.layers, cfg.heads,
                    cfg.d_k, cfg.d_v, cfg.R, cfg.W, factors)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(fn: str, rc: int) -> None:
    if rc != 0:
        raise SeedError(fn, rc)


def _check_state(dims: "Dims", state: "State") -> None:
    """The C ABI sees only pointers: check here that the state's tensors have the
    element types and sizes the dims describe (U and V in the factor format)."""
    B, L, H, m = dims.batch, dims.layers, dims.heads, dims.m
    slen = dims.d_k if dims.form == SEED_KDA else (m + 3) // 4 * 4
    want = {"a": (torch.float32, B * L * H * dims.d_k),
            "U": (FACTOR_DTYPES[dims.factors], B * L * H * m * dims.d_k),
            "V": (FACTOR_DTYPES[dims.factors], B * L * H * m * dims.d_v),
            "scale": (torch.float32, B * L * H * slen),
            "ncols": (torch.int32, B * L * H),
            "vbar": (torch.float32, L * H * dims.d_v)}
    for name, (dtype, n) in want.items():
        t = getattr(state, name)
        if t.dtype != dtype or t.numel() < n:
            raise ValueError(f"state.{name}: expected {dtype} with at least {n} elements, got {t.dtype} "
                             f"with {t.numel()}")


@dataclass
class State:
    """Device tensors of the stored state (layouts as in seed.h)."""
    a: torch.Tensor          # [B][L][H][d_k]
    U: torch.Tensor          # [B][L][H][R+W][d_k], element type dims.factor_dtype
    V: torch.Tensor          # [B][L][H][R+W][d_v], same
    scale: torch.Tensor      # [B][L][H][ceil4(R+W)] (GDN, Mamba-2) or [B][L][H][d_k] (KDA)
    ncols: torch.Tensor      # [B][L][H] int32
    vbar: torch.Tensor       # [L][H][d_v]

    def c(self) -> _lib.seed_state:
        return _lib.seed_state(_ptr(self.a), _ptr(self.U), _ptr(self.V), _ptr(self.scale),
                               _ptr(self.ncols), _ptr(self.vbar))

    @staticmethod
    def allocate(dims: Dims, vbar: torch.Tensor, device=None) -> "State":
        dev = vbar.device if device is None else device
        B, L, H = dims.batch, dims.layers, dims.heads
        slen = dims.d_k if dims.form == SEED_KDA else (dims.m + 3) // 4 * 4
        f32 = dict(dtype=torch.float32, device=dev)
        fac = dict(dtype=FACTOR_DTYPES[dims.factors], device=dev)
        return State(a=torch.zeros(B, L, H, dims.d_k, **f32),
                     U=torch.zeros(B, L, H, dims.m, dims.d_k, **fac),
                     V=torch.zeros(B, L, H, dims.m, dims.d_v, **fac),
                     scale=torch.ones(B, L, H, slen, **f32),
                     ncols=torch.zeros(B, L, H, dtype=torch.int32, device=dev),
                     vbar=vbar)

    def state_dict(self) -> dict:
        return {"a": self.a, "U": self.U, "V": self.V, "scale": self.scale, "ncols": self.ncols}

    def load_state_dict(self, sd: dict) -> None:
        for k in ("a", "U", "V", "scale", "ncols"):
            getattr(self, k).copy_(sd[k])


class Workspace:
    """The device workspace (status word) every call needs."""

    def __init__(self, dims: Dims, device="cuda"):
        lib = _lib.load()
        d = dims.c()
        self.nbytes = int(lib.seed_workspace_bytes(ctypes.byref(d)))
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        _check("seed_workspace_init", lib.seed_workspace_init(_ptr(self.buf), self.nbytes, _stream(None)))

    @property
    def ptr(self) -> int:
        return self.buf.data_ptr()


def seed_scale_len(dims: Dims) -> int:
    return int(_lib.load().seed_scale_len(ctypes.byref(dims.c())))


def seed_workspace_bytes(dims: Dims) -> int:
    return int(_lib.load().seed_workspace_bytes(ctypes.byref(dims.c())))


def seed_state_init_from_dense(dims: Dims, state: State, layer: int, S_dense: torch.Tensor,
                               ws: Workspace, sigma_out: torch.Tensor | None = None, stream=None) -> None:
    _check_state(dims, state)
    d, s = dims.c(), state.c()
    _check("seed_state_init_from_dense", _lib.load().seed_state_init_from_dense(
        ctypes.byref(d), ctypes.byref(s), layer, _ptr(S_dense), _ptr(sigma_out), ws.ptr, ws.nbytes,
        _stream(stream)))


def seed_decode_step(dims: Dims, state: State, layer: int, q, k, v, alpha, beta, o,
                     ws: Workspace, stream=None) -> None:
    _check_state(dims, state)
    d, s = dims.c(), state.c()
    _check("seed_decode_step", _lib.load().seed_decode_step(
        ctypes.byref(d), ctypes.byref(s), layer, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
        _ptr(o), ws.ptr, ws.nbytes, _stream(stream)))


def seed_decode_step_overlapped(dims: Dims, state: State, layer: int, q, k, v, alpha, beta, o,
                                ws: Workspace, stream=None) -> None:
    """seed_decode_step for a stream whose previous launch does not write this layer's
    state (e.g. another layer's step): the step may begin streaming the state while
    that launch finishes, and reads its inputs after it."""
    _check_state(dims, state)
    d, s = dims.c(), state.c()
    _check("seed_decode_step_overlapped", _lib.load().seed_decode_step_overlapped(
        ctypes.byref(d), ctypes.byref(s), layer, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
        _ptr(o), ws.ptr, ws.nbytes, _stream(stream)))


def seed_decode_step_noalloc(dims: Dims, state: State, layer: int, q, k, v, alpha, beta, o,
                             status_out: torch.Tensor | None = None, stream=None) -> None:
    """seed_decode_step with the library's own fixed device workspace; status_out, if
    given, is a device int32/uint32 tensor of one element that receives the flags."""
    _check_state(dims, state)
    d, s = dims.c(), state.c()
    _check("seed_decode_step_noalloc", _lib.load().seed_decode_step_noalloc(
        ctypes.byref(d), ctypes.byref(s), layer, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
        _ptr(o), _ptr(status_out), _stream(stream)))


def seed_decode_step_compress(dims: Dims, state: State, layer: int, q, k, v, alpha, beta, o,
                              ws: Workspace, sigma_out: torch.Tensor | None = None, stream=None) -> None:
    """seed_decode_step fused with the compression of the units the step brings to
    R + W columns; sigma_out [B * H][R] (rows of compressed units written)."""
    _check_state(dims, state)
    d, s = dims.c(), state.c()
    _check("seed_decode_step_compress", _lib.load().seed_decode_step_compress(
        ctypes.byref(d), ctypes.byref(s), layer, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
        _ptr(o), _ptr(sigma_out), ws.ptr, ws.nbytes, _stream(stream)))


def seed_noalloc_workspace_bytes() -> int:
    return int(_lib.load().seed_noalloc_workspace_bytes())


def seed_compress(dims: Dims, state: State, layer: int, ws: Workspace,
                  sigma_out: torch.Tensor | None = None, stream=None) -> None:
    _check_state(dims, state)
    d, s = dims.c(), state.c()
    _check("seed_compress", _lib.load().seed_compress(
        ctypes.byref(d), ctypes.byref(s), layer, _ptr(sigma_out), ws.ptr, ws.nbytes, _stream(stream)))


def seed_state_to_dense(dims: Dims, state: State, layer: int, S_out: torch.Tensor, ws: Workspace,
                        units: torch.Tensor | None = None, stream=None) -> None:
    _check_state(dims, state)
    d, s = dims.c(), state.c()
    n = 0 if units is None else int(units.numel())
    _check("seed_state_to_dense", _lib.load().seed_state_to_dense(
        ctypes.byref(d), ctypes.byref(s), layer, _ptr(units), n, _ptr(S_out), ws.ptr, ws.nbytes,
        _stream(stream)))


def seed_state_energy(dims: Dims, state: State, layer: int, out: torch.Tensor, ws: Workspace,
                      units: torch.Tensor | None = None, stream=None) -> None:
    """out [n][4]: sink energy, content energy, cross term, total (see seed.h)."""
    _check_state(dims, state)
    d, s = dims.c(), state.c()
    n = 0 if units is None else int(units.numel())
    _check("seed_state_energy", _lib.load().seed_state_energy(
        ctypes.byref(d), ctypes.byref(s), layer, _ptr(units), n, _ptr(out), ws.ptr, ws.nbytes,
        _stream(stream)))


def seed_state_spectrum(dims: Dims, state: State, layer: int, sigma_state: torch.Tensor,
                        sigma_content: torch.Tensor, cos_top: torch.Tensor, ranks: torch.Tensor,
                        ws: Workspace, units: torch.Tensor | None = None, stream=None) -> None:
    """sigma_state, sigma_content [n][R+W+1], cos_top [n] (float32); ranks [n][2] int32 (see seed.h)."""
    _check_state(dims, state)
    if ranks.dtype != torch.int32:
        raise ValueError("ranks must be int32")
    d, s = dims.c(), state.c()
    n = 0 if units is None else int(units.numel())
    _check("seed_state_spectrum", _lib.load().seed_state_spectrum(
        ctypes.byref(d), ctypes.byref(s), layer, _ptr(units), n, _ptr(sigma_state), _ptr(sigma_content),
        _ptr(cos_top), _ptr(ranks), ws.ptr, ws.nbytes, _stream(stream)))


def seed_dense_step(dims: Dims, S: torch.Tensor, layer: int, q, k, v, alpha, beta, o,
                    ws: Workspace, stream=None) -> None:
    d = dims.c()
    _check("seed_dense_step", _lib.load().seed_dense_step(
        ctypes.byref(d), _ptr(S), layer, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(o),
        ws.ptr, ws.nbytes, _stream(stream)))


def seed_get_status(ws: Workspace, stream=None) -> int:
    flags = _lib.c_uint32(0)
    _check("seed_get_status", _lib.load().seed_get_status(ws.ptr, _stream(stream), ctypes.byref(flags)))
    return int(flags.value)


def seed_get_diagnostics(ws: Workspace, stream=None) -> dict:
    c = (_lib.c_uint32 * 6)()
    _check("seed_get_diagnostics", _lib.load().seed_get_diagnostics(ws.ptr, _stream(stream), c))
    return {"compress_sweeps": c[0], "householder_units": c[1], "convert_sweeps": c[2],
            "convert_units": c[3], "cholqr_units": c[4], "cholqr_declined": c[5],
            "compress_units": c[1] + c[4]}


def seed_debug_wait_fault(ws: Workspace, enable: bool, stream=None) -> None:
    _check("seed_debug_wait_fault",
           _lib.load().seed_debug_wait_fault(ws.ptr, ws.nbytes, 1 if enable else 0, _stream(stream)))


# ------------------------------------------------------------------ synthetic workloads

def synth_key(cfg, b0: int = 0) -> _lib.seed_synth_key:
    return _lib.seed_synth_key(cfg.seed, cfg.cid, 1 if cfg.vbar_unit else 0, b0)


def seed_synth_vbar(dims: Dims, key, vbar: torch.Tensor, stream=None) -> None:
    d = dims.c()
    _check("seed_synth_vbar", _lib.load().seed_synth_vbar(ctypes.byref(d), key, _ptr(vbar), _stream(stream)))


def seed_synth_token_inputs(dims: Dims, key, phase: int, t: int, layer: int, vbar, q, k, v, alpha, beta,
                            stream=None) -> None:
    d = dims.c()
    _check("seed_synth_token_inputs", _lib.load().seed_synth_token_inputs(
        ctypes.byref(d), key, phase, t, layer, _ptr(vbar), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
        _ptr(beta), _stream(stream)))


def seed_synth_dense_prefill(dims: Dims, key, n_tokens: int, layer: int, vbar, S_out, stream=None) -> None:
    d = dims.c()
    _check("seed_synth_dense_prefill", _lib.load().seed_synth_dense_prefill(
        ctypes.byref(d), key, n_tokens, layer, _ptr(vbar), _ptr(S_out), _stream(stream)))


# ------------------------------------------------------------------ convenience (allocation only)

def alloc_step_inputs(dims: Dims, device="cuda", with_q: bool = True) -> dict:
    """Empty per-layer step tensors: q, k [B][H][d_k], v, o [B][H][d_v], alpha, beta."""
    B, H = dims.batch, dims.heads
    f = dict(dtype=torch.float32, device=device)
    out = {"k": torch.empty(B, H, dims.d_k, **f), "v": torch.empty(B, H, dims.d_v, **f),
           "beta": torch.empty(B, H, **f), "o": torch.empty(B, H, dims.d_v, **f)}
    out["q"] = torch.empty(B, H, dims.d_k, **f) if with_q else None
    out["alpha"] = (torch.empty(B, H, dims.d_k, **f) if dims.form == SEED_KDA
                    else torch.empty(B, H, **f))
    return out
