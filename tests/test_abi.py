"""The C ABI without a GPU: libseed.so loads, exports every function the headers
declare, and rejects bad arguments on the host before anything is enqueued."""

import ctypes
import glob
import os
import re

import pytest

from rank_recurrent_state_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*[A-Za-z_][\w\s\*]*?\b(seed_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return names


def test_headers_declare_the_entry_points():
    names = _declared_functions()
    for n in ("seed_state_init_from_dense", "seed_decode_step", "seed_compress",
              "seed_state_to_dense", "seed_dense_step", "seed_get_status", "seed_workspace_bytes",
              "seed_synth_token_inputs", "seed_synth_dense_prefill", "seed_synth_vbar"):
        assert n in names


def test_library_exports_every_declared_function(lib):
    names = _declared_functions()
    assert names
    for n in sorted(names):
        assert hasattr(lib, n), n
        assert n in _lib.SIGNATURES, f"binding lacks {n}"


def _dims(**kw):
    base = dict(form=0, batch=2, layers=3, heads=4, d_k=128, d_v=128, R=16, W=16)
    base.update(kw)
    return _lib.seed_dims(**base)


A = 0x10000          # fake, aligned device addresses: never dereferenced on error paths
MIS = 0x10004        # misaligned


def _state(**kw):
    base = dict(a=A, U=A, V=A, scale=A, ncols=A, vbar=A)
    base.update(kw)
    return _lib.seed_state(**base)


def test_status_strings(lib):
    assert lib.seed_status_string(0) == b"ok"
    for code in (-1, -2, -3, -4, -5):
        assert lib.seed_status_string(code) != b"unknown status"


def test_scale_len_and_workspace(lib):
    d = _dims()
    assert lib.seed_scale_len(ctypes.byref(d)) == 32
    dk = _dims(form=1)
    assert lib.seed_scale_len(ctypes.byref(dk)) == 128
    assert lib.seed_workspace_bytes(ctypes.byref(d)) >= 4
    bad = _dims(d_k=48)
    assert lib.seed_scale_len(ctypes.byref(bad)) == -1


@pytest.mark.parametrize("dims,code", [
    (None, -1),
    (_dims(form=3), -1),
    (_dims(factors=3), -1),                     # no such factor format
    (_dims(factors=-1), -1),
    (_dims(batch=0), -1),
    (_dims(R=0), -1),
    (_dims(d_k=48), -2),
    (_dims(d_k=256, d_v=256), -2),
    (_dims(d_k=16, d_v=16, R=8, W=16), -2),     # R + W > d
    (_dims(R=64, W=64), -2),                    # R + W > SEED_MAX_COLS
])
@pytest.mark.parametrize("entry", ["seed_decode_step", "seed_decode_step_overlapped"])
def test_decode_step_rejects_bad_dims(lib, dims, code, entry):
    d = ctypes.byref(dims) if dims is not None else None
    s = _state()
    rc = getattr(lib, entry)(d, ctypes.byref(s), 0, A, A, A, A, A, A, A, 256, None)
    assert rc == code


@pytest.mark.parametrize("entry", ["seed_decode_step", "seed_decode_step_overlapped"])
def test_decode_step_rejects_bad_pointers_and_layer(lib, entry):
    d, s = _dims(), _state()
    call = lambda layer=0, st=s, q=A, ws=A, wsb=256: getattr(lib, entry)(  # noqa: E731
        ctypes.byref(d), ctypes.byref(st), layer, q, A, A, A, A, A, ws, wsb, None)
    assert call(layer=3) == -1
    assert call(layer=-1) == -1                  # all layers is not a decode step
    assert call(q=None) == -1
    assert call(q=MIS) == -3
    assert call(st=_state(U=MIS)) == -3
    assert call(st=_state(ncols=None)) == -1
    assert call(ws=None) == -5
    assert call(wsb=8) == -5


def test_other_entry_points_validate(lib):
    d, s = _dims(), _state()
    assert lib.seed_compress(ctypes.byref(d), ctypes.byref(s), 5, None, A, 256, None) == -1
    assert lib.seed_compress(ctypes.byref(d), ctypes.byref(s), 0, MIS, A, 256, None) == -3
    assert lib.seed_state_init_from_dense(ctypes.byref(d), ctypes.byref(s), -1, None, None, A, 256,
                                          None) == -1
    assert lib.seed_state_to_dense(ctypes.byref(d), ctypes.byref(s), 0, A, 10**6, A, A, 256, None) == -1
    assert lib.seed_state_to_dense(ctypes.byref(d), ctypes.byref(s), 0, A, 0, A, A, 256, None) == 0
    assert lib.seed_dense_step(ctypes.byref(d), MIS, 0, A, A, A, A, A, A, A, 256, None) == -3
    flags = _lib.c_uint32()
    assert lib.seed_get_status(None, None, ctypes.byref(flags)) == -5
    assert lib.seed_get_status(A, None, None) == -1
    key = _lib.seed_synth_key(0, 0, 0, 0)
    assert lib.seed_synth_token_inputs(ctypes.byref(d), key, 3, 0, 0, A, A, A, A, A, A, None) == -1
    assert lib.seed_synth_dense_prefill(ctypes.byref(d), key, -1, 0, A, A, None) == -1
    bad_key = _lib.seed_synth_key(0, 0, 0, -1)
    assert lib.seed_synth_dense_prefill(ctypes.byref(d), bad_key, 4, 0, A, A, None) == -1


def test_fused_decode_compress_validates(lib):
    d, s = _dims(), _state()
    call = lambda layer=0, q=A, sig=None, wsb=256: lib.seed_decode_step_compress(  # noqa: E731
        ctypes.byref(d), ctypes.byref(s), layer, q, A, A, A, A, A, sig, A, wsb, None)
    assert call(layer=-1) == -1                  # one layer per call
    assert call(layer=3) == -1
    assert call(q=MIS) == -3
    assert call(sig=MIS) == -3
    assert call(wsb=8) == -5
    bad = _dims(factors=7)
    assert lib.seed_decode_step_compress(ctypes.byref(bad), ctypes.byref(s), 0, A, A, A, A, A, A, None, A, 256,
                                         None) == -1


def test_noalloc_decode_step_validates_before_touching_the_device(lib):
    d, s = _dims(), _state()
    assert lib.seed_noalloc_workspace_bytes() >= lib.seed_workspace_bytes(ctypes.byref(d))
    assert lib.seed_decode_step_noalloc(None, ctypes.byref(s), 0, A, A, A, A, A, A, None, None) == -1
    assert lib.seed_decode_step_noalloc(ctypes.byref(d), ctypes.byref(s), 0, A, A, A, A, A, A,
                                        0x10002, None) == -3


def test_headers_compile_as_c_and_link(lib, tmp_path):
    """A plain C99 program includes both headers, links against libseed.so and calls
    entry points whose argument checks run on the host (no device needed)."""
    import shutil
    import subprocess
    from rank_recurrent_state_b200 import build as b
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(r"""
#include <stdio.h>
#include "seed.h"
#include "seed_synth.h"
int main(void) {
  seed_dims d = {SEED_GDN, 2, 3, 4, 128, 128, 16, 16, SEED_FACTORS_F16};
  seed_state s = {0};
  if (seed_scale_len(&d) != 32) return 1;
  if (seed_workspace_bytes(&d) < 4) return 2;
  if (seed_decode_step(&d, &s, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0) != SEED_ERR_INVALID_ARG) return 3;
  d.factors = 9;
  if (seed_scale_len(&d) != -1) return 4;
  printf("%s\n", seed_status_string(SEED_ERR_SHAPE));
  return 0;
}
""")
    exe = tmp_path / "abi"
    libdir = os.path.dirname(b.LIB)
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                        "-o", str(exe), "-L", libdir, "-lseed", f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stderr)
    assert r.stdout.strip()


def test_binding_checks_state_types_before_calling():
    """The binding rejects a state whose factor tensors do not have the dims' element
    type (the C ABI cannot see it) before anything reaches the library."""
    import torch
    from rank_recurrent_state_b200 import seed as S
    d = S.Dims(S.SEED_GDN, 2, 1, 2, 64, 64, 8, 8, S.SEED_FACTORS_F16)
    vbar = torch.ones(1, 2, 64)
    st = S.State.allocate(d, vbar, device="cpu")
    assert st.U.dtype == torch.float16 and st.V.dtype == torch.float16
    S._check_state(d, st)                                   # matches: no error
    st32 = S.State.allocate(S.Dims(S.SEED_GDN, 2, 1, 2, 64, 64, 8, 8), vbar, device="cpu")
    with pytest.raises(ValueError, match="state.U"):
        S.seed_compress(d, st32, S.SEED_ALL_LAYERS, None)
    small = S.State.allocate(S.Dims(S.SEED_GDN, 1, 1, 2, 64, 64, 8, 8, S.SEED_FACTORS_F16), vbar, device="cpu")
    with pytest.raises(ValueError, match="state.a"):
        S.seed_decode_step(d, small, 0, None, None, None, None, None, None, None)


def test_oracle_and_product_path_share_no_code():
    """The package never imports the oracle, the oracle never imports the package or
    loads the library; the one module both use is the seeded input generator."""
    import ast
    pkg = os.path.join(ROOT, "rank_recurrent_state_b200")
    for path in glob.glob(os.path.join(pkg, "*.py")):
        tree = ast.parse(open(path).read())
        for node in ast.walk(tree):
            names = ([a.name for a in node.names] if isinstance(node, ast.Import)
                     else [node.module or ""] if isinstance(node, ast.ImportFrom) else [])
            assert not any(n.split(".")[0] == "oracle" for n in names), path
    for path in glob.glob(os.path.join(ROOT, "rank_recurrent_state_b200", "csrc", "*")):
        assert "oracle" not in open(path).read().lower(), path
    for path in glob.glob(os.path.join(ROOT, "oracle", "*.py")):
        text = open(path).read()
        assert "rank_recurrent_state_b200" not in text and "libseed" not in text, path


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    """Without libseed.so the binding raises; there is no CPU path to fall back to."""
    monkeypatch.setattr(_lib, "_LIB", None)
    with pytest.raises(ImportError, match="no CPU fallback"):
        _lib.load(str(tmp_path / "libseed.so"))
