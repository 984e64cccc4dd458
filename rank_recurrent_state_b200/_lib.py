"""ctypes view of libseed.so (include/seed.h, include/seed_synth.h).

Loading fails loudly when the library has not been built: there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libseed.so")

c_int32 = ctypes.c_int32
c_uint32 = ctypes.c_uint32
c_void_p = ctypes.c_void_p
c_size_t = ctypes.c_size_t
c_float_p = ctypes.POINTER(ctypes.c_float)


class seed_dims(ctypes.Structure):
    _fields_ = [("form", c_int32), ("batch", c_int32), ("layers", c_int32), ("heads", c_int32),
                ("d_k", c_int32), ("d_v", c_int32), ("R", c_int32), ("W", c_int32), ("factors", c_int32)]


class seed_state(ctypes.Structure):
    _fields_ = [("a", c_void_p), ("U", c_void_p), ("V", c_void_p), ("scale", c_void_p),
                ("ncols", c_void_p), ("vbar", c_void_p)]


class seed_synth_key(ctypes.Structure):
    _fields_ = [("seed", c_uint32), ("workload", c_uint32), ("vbar_unit", c_int32), ("b0", c_int32)]


# name -> (restype, argtypes)
SIGNATURES = {
    "seed_scale_len": (c_int32, [ctypes.POINTER(seed_dims)]),
    "seed_workspace_bytes": (c_size_t, [ctypes.POINTER(seed_dims)]),
    "seed_workspace_init": (ctypes.c_int, [c_void_p, c_size_t, c_void_p]),
    "seed_state_init_from_dense": (ctypes.c_int, [ctypes.POINTER(seed_dims), ctypes.POINTER(seed_state),
                                                  c_int32, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "seed_decode_step": (ctypes.c_int, [ctypes.POINTER(seed_dims), ctypes.POINTER(seed_state), c_int32,
                                        c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                        c_void_p, c_size_t, c_void_p]),
    "seed_decode_step_overlapped": (ctypes.c_int, [ctypes.POINTER(seed_dims), ctypes.POINTER(seed_state), c_int32,
                                                   c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                                   c_void_p, c_size_t, c_void_p]),
    "seed_compress": (ctypes.c_int, [ctypes.POINTER(seed_dims), ctypes.POINTER(seed_state), c_int32,
                                     c_void_p, c_void_p, c_size_t, c_void_p]),
    "seed_decode_step_compress": (ctypes.c_int, [ctypes.POINTER(seed_dims), ctypes.POINTER(seed_state), c_int32,
                                                 c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                                 c_void_p, c_void_p, c_size_t, c_void_p]),
    "seed_state_to_dense": (ctypes.c_int, [ctypes.POINTER(seed_dims), ctypes.POINTER(seed_state), c_int32,
                                           c_void_p, c_int32, c_void_p, c_void_p, c_size_t, c_void_p]),
    "seed_state_energy": (ctypes.c_int, [ctypes.POINTER(seed_dims), ctypes.POINTER(seed_state), c_int32,
                                         c_void_p, c_int32, c_void_p, c_void_p, c_size_t, c_void_p]),
    "seed_state_spectrum": (ctypes.c_int, [ctypes.POINTER(seed_dims), ctypes.POINTER(seed_state), c_int32,
                                           c_void_p, c_int32, c_void_p, c_void_p, c_void_p, c_void_p,
                                           c_void_p, c_size_t, c_void_p]),
    "seed_dense_step": (ctypes.c_int, [ctypes.POINTER(seed_dims), c_void_p, c_int32, c_void_p, c_void_p,
                                       c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                       c_void_p]),
    "seed_get_status": (ctypes.c_int, [c_void_p, c_void_p, ctypes.POINTER(c_uint32)]),
    "seed_get_diagnostics": (ctypes.c_int, [c_void_p, c_void_p, ctypes.POINTER(c_uint32)]),
    "seed_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "seed_debug_wait_fault": (ctypes.c_int, [c_void_p, c_size_t, c_int32, c_void_p]),
    "seed_synth_vbar": (ctypes.c_int, [ctypes.POINTER(seed_dims), seed_synth_key, c_void_p, c_void_p]),
    "seed_synth_token_inputs": (ctypes.c_int, [ctypes.POINTER(seed_dims), seed_synth_key, c_int32, c_int32,
                                               c_int32, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                               c_void_p, c_void_p]),
    "seed_synth_dense_prefill": (ctypes.c_int, [ctypes.POINTER(seed_dims), seed_synth_key, c_int32, c_int32,
                                                c_void_p, c_void_p, c_void_p]),
    "seed_noalloc_workspace_bytes": (c_size_t, []),
    "seed_decode_step_noalloc": (ctypes.c_int, [ctypes.POINTER(seed_dims), ctypes.POINTER(seed_state),
                                                c_int32, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                                c_void_p, c_void_p, c_void_p]),
}

_LIB = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libseed.so and declare every entry point; raises if it is missing."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m rank_recurrent_state_b200.build` "
                          "(the decode path has no CPU fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = lib
    return lib
