"""C-ABI library: it loads, exports every symbol the public header declares,
and rejects bad arguments on the host before touching a device (no GPU)."""
from __future__ import annotations

import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "paged_kv_cache_412_b200", "libpkv.so")


def _declared_functions():
    names = set()
    for hdr in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(hdr).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b(pkv_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        from paged_kv_cache_412_b200 import build
        build.build()
    return ctypes.CDLL(LIB)


def test_header_declares_the_hot_path_calls():
    names = _declared_functions()
    for n in ("pkv_kv_cache_write", "pkv_paged_attention_decode", "pkv_copy_blocks",
              "pkv_paged_attention_decode_append", "pkv_decode_workspace_bytes",
              "pkv_get_device_error", "pkv_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings(lib):
    lib.pkv_status_string.restype = ctypes.c_char_p
    assert lib.pkv_status_string(0) == b"PKV_OK"
    assert b"WORKSPACE" in lib.pkv_status_string(3)
    assert b"UNKNOWN" in lib.pkv_status_string(99)
    assert lib.pkv_version() >= 100


def test_binding_imports_and_names_match(lib):
    import paged_kv_cache_412_b200 as pkv
    assert os.path.samefile(pkv.LIB_PATH, LIB)
    for fn in ("kv_cache_write", "paged_attention_decode", "copy_blocks"):
        assert callable(getattr(pkv, fn))


# Host validation paths that return before any CUDA call.
V = ctypes.c_void_p
DUMMY = V(0x10000)


def _write(lib, **kw):
    a = dict(k=DUMMY, v=DUMMY, slots=DUMMY, kc=DUMMY, vc=DUMMY, T=4, Hkv=2, d=64, bs=16, NB=8,
             dt=1)
    a.update(kw)
    f = lib.pkv_kv_cache_write
    f.argtypes = [V, V, V, V, V, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                  ctypes.c_int32, ctypes.c_int, V]
    return f(a["k"], a["v"], a["slots"], a["kc"], a["vc"], a["T"], a["Hkv"], a["d"], a["bs"],
             a["NB"], a["dt"], None)


def test_write_rejects_bad_args(lib):
    assert _write(lib, T=-1) == 1
    assert _write(lib, bs=12) == 1          # not a power of two
    assert _write(lib, bs=512) == 1         # too large
    assert _write(lib, dt=7) == 1           # unknown dtype
    assert _write(lib, d=96) == 2           # unsupported head_dim
    assert _write(lib, T=0) == 0            # nothing to do
    assert _write(lib, k=None) == 1         # null pointer
    assert _write(lib, kc=V(0x10004)) == 1  # misaligned cache


def _decode(lib, **kw):
    a = dict(q=DUMMY, kc=DUMMY, vc=DUMMY, bt=DUMMY, sl=DUMMY, bs=16, scale=0.125, out=DUMMY,
             B=2, Hq=8, Hkv=2, d=128, maxb=4, NB=8, maxL=64, qdt=1, kvdt=1, odt=1, ks=None,
             vs=None, P=0, ws=DUMMY, wsb=1 << 20)
    a.update(kw)
    f = lib.pkv_paged_attention_decode
    i32 = ctypes.c_int32
    f.argtypes = [V, V, V, V, V, i32, ctypes.c_float, V, i32, i32, i32, i32, i32, i32, i32,
                  ctypes.c_int, ctypes.c_int, ctypes.c_int, V, V, i32, V, ctypes.c_size_t, V]
    return f(a["q"], a["kc"], a["vc"], a["bt"], a["sl"], a["bs"], a["scale"], a["out"], a["B"],
             a["Hq"], a["Hkv"], a["d"], a["maxb"], a["NB"], a["maxL"], a["qdt"], a["kvdt"],
             a["odt"], a["ks"], a["vs"], a["P"], a["ws"], a["wsb"], None)


def test_decode_rejects_bad_args(lib):
    assert _decode(lib, Hq=6, Hkv=4) == 1       # Hq % Hkv != 0
    assert _decode(lib, bs=24) == 1             # not a power of two
    assert _decode(lib, d=80) == 2              # unsupported head_dim
    assert _decode(lib, qdt=0, kvdt=1) == 1     # dtype mismatch
    assert _decode(lib, odt=2) == 2             # fp8 output not supported
    assert _decode(lib, P=48) == 1              # partition not a multiple of 32
    assert _decode(lib, scale=float("nan")) == 1
    assert _decode(lib, B=-1) == 1
    assert _decode(lib, B=0) == 0               # empty batch: nothing to do
    assert _decode(lib, q=None) == 1
    assert _decode(lib, maxb=0) == 1


def _decode_append(lib, **kw):
    a = dict(q=DUMMY, kn=V(0x20000), vn=V(0x30000), kc=DUMMY, vc=DUMMY, bt=DUMMY, sl=DUMMY,
             bs=16, scale=0.125, out=DUMMY, B=2, Hq=8, Hkv=2, d=128, maxb=4, NB=8, maxL=64,
             odt=1, P=0, ws=DUMMY, wsb=1 << 20)
    a.update(kw)
    f = lib.pkv_paged_attention_decode_append
    i32 = ctypes.c_int32
    f.argtypes = [V, V, V, V, V, V, V, i32, ctypes.c_float, V, i32, i32, i32, i32, i32, i32, i32,
                  ctypes.c_int, i32, V, ctypes.c_size_t, V]
    return f(a["q"], a["kn"], a["vn"], a["kc"], a["vc"], a["bt"], a["sl"], a["bs"], a["scale"],
             a["out"], a["B"], a["Hq"], a["Hkv"], a["d"], a["maxb"], a["NB"], a["maxL"], a["odt"],
             a["P"], a["ws"], a["wsb"], None)


def test_decode_append_rejects_bad_args(lib):
    """Checked on the host before any device call (so no GPU is needed)."""
    assert _decode_append(lib, kn=None) == 1          # a request has no new K row
    assert _decode_append(lib, vn=None) == 1
    assert _decode_append(lib, kn=V(0x20002)) == 1    # not on a 16-byte boundary
    assert _decode_append(lib, bs=1) == 2             # no tensor-core path for 1-row blocks
    assert _decode_append(lib, d=256) == 2
    assert _decode_append(lib, Hq=6, Hkv=4) == 1      # the decode's own checks still apply
    assert _decode_append(lib, B=0, kn=None, vn=None) == 0  # empty batch: nothing to do


def _copy(lib, **kw):
    a = dict(kc=DUMMY, vc=DUMMY, bm=DUMMY, n=3, Hkv=2, d=64, bs=16, NB=8, dt=1)
    a.update(kw)
    f = lib.pkv_copy_blocks
    i32 = ctypes.c_int32
    f.argtypes = [V, V, V, i32, i32, i32, i32, i32, ctypes.c_int, V]
    return f(a["kc"], a["vc"], a["bm"], a["n"], a["Hkv"], a["d"], a["bs"], a["NB"], a["dt"], None)


def test_copy_rejects_bad_args(lib):
    assert _copy(lib, n=-2) == 1
    assert _copy(lib, bs=3) == 1
    assert _copy(lib, d=32) == 2
    assert _copy(lib, n=0) == 0
    assert _copy(lib, bm=None) == 1
    assert _copy(lib, bm=V(0x10004)) == 1


def test_get_device_error_needs_output_pointer(lib):
    f = lib.pkv_get_device_error
    f.argtypes = [V, V]
    assert f(None, None) == 1


def _write_fp8(lib, **kw):
    a = dict(k=DUMMY, v=DUMMY, slots=DUMMY, kc=DUMMY, vc=DUMMY, ks=DUMMY, vs=DUMMY, T=4, Hkv=2,
             d=128, bs=16, NB=8)
    a.update(kw)
    f = lib.pkv_kv_cache_write_fp8
    i32 = ctypes.c_int32
    f.argtypes = [V, V, V, V, V, V, V, i32, i32, i32, i32, i32, V]
    return f(a["k"], a["v"], a["slots"], a["kc"], a["vc"], a["ks"], a["vs"], a["T"], a["Hkv"],
             a["d"], a["bs"], a["NB"], None)


def test_fp8_write_rejects_bad_args(lib):
    assert _write_fp8(lib, T=-1) == 1
    assert _write_fp8(lib, NB=0) == 1
    assert _write_fp8(lib, d=96) == 2           # unsupported head_dim
    assert _write_fp8(lib, T=0) == 0            # nothing to do
    assert _write_fp8(lib, ks=None) == 1        # the per-head scales are required
    assert _write_fp8(lib, vs=None) == 1
    assert _write_fp8(lib, k=V(0x10008)) == 1   # misaligned input rows


def _prefix(lib, **kw):
    a = dict(q=DUMMY, kc=DUMMY, vc=DUMMY, bt=DUMMY, sl=DUMMY, bs=16, scale=0.125, out=DUMMY,
             B=2, Hq=8, Hkv=2, d=128, maxb=4, NB=8, maxL=64, qdt=1, kvdt=1, odt=1, po=DUMMY,
             pl=DUMMY, npfx=1, maxm=2, maxpl=64, ws=DUMMY, wsb=1 << 20)
    a.update(kw)
    f = lib.pkv_paged_attention_decode_prefix
    i32 = ctypes.c_int32
    f.argtypes = [V, V, V, V, V, i32, ctypes.c_float, V, i32, i32, i32, i32, i32, i32, i32,
                  ctypes.c_int, ctypes.c_int, ctypes.c_int, V, V, i32, i32, i32, V,
                  ctypes.c_size_t, V]
    return f(a["q"], a["kc"], a["vc"], a["bt"], a["sl"], a["bs"], a["scale"], a["out"], a["B"],
             a["Hq"], a["Hkv"], a["d"], a["maxb"], a["NB"], a["maxL"], a["qdt"], a["kvdt"],
             a["odt"], a["po"], a["pl"], a["npfx"], a["maxm"], a["maxpl"], a["ws"], a["wsb"],
             None)


def test_prefix_decode_rejects_bad_args(lib):
    # the checks the prefix-aware call shares with the plain decode (made
    # before any device is touched)
    assert _prefix(lib, Hq=6, Hkv=4) == 1
    assert _prefix(lib, bs=24) == 1
    assert _prefix(lib, d=80) == 2
    assert _prefix(lib, odt=2) == 2
    assert _prefix(lib, q=None) == 1
    assert _prefix(lib, out=V(0x10001)) == 1
    assert _prefix(lib, B=0) == 0


def _swap(lib, **kw):
    a = dict(sk=DUMMY, sv=DUMMY, dk=DUMMY, dv=DUMMY, bm=DUMMY, n=3, sNB=8, dNB=8, Hkv=2, d=64,
             bs=16, dt=1)
    a.update(kw)
    f = lib.pkv_swap_blocks
    i32 = ctypes.c_int32
    f.argtypes = [V, V, V, V, V, i32, i32, i32, i32, i32, i32, ctypes.c_int, V]
    return f(a["sk"], a["sv"], a["dk"], a["dv"], a["bm"], a["n"], a["sNB"], a["dNB"], a["Hkv"],
             a["d"], a["bs"], a["dt"], None)


def test_swap_rejects_bad_args(lib):
    assert _swap(lib, n=-1) == 1
    assert _swap(lib, sNB=0) == 1
    assert _swap(lib, dt=7) == 1                # unknown dtype
    assert _swap(lib, d=96) == 2
    assert _swap(lib, n=0) == 0                 # nothing to do
    assert _swap(lib, bm=None) == 1
    assert _swap(lib, dk=None) == 1


def _decode_noalloc(lib, **kw):
    a = dict(q=DUMMY, kc=DUMMY, vc=DUMMY, bt=DUMMY, sl=DUMMY, bs=16, scale=0.125, out=DUMMY,
             B=2, Hq=8, Hkv=2, d=128, maxb=4, NB=8, maxL=64, qdt=1, kvdt=1, odt=1, ks=None,
             vs=None, P=0)
    a.update(kw)
    f = lib.pkv_paged_attention_decode_noalloc
    i32 = ctypes.c_int32
    f.argtypes = [V, V, V, V, V, i32, ctypes.c_float, V, i32, i32, i32, i32, i32, i32, i32,
                  ctypes.c_int, ctypes.c_int, ctypes.c_int, V, V, i32, V]
    return f(a["q"], a["kc"], a["vc"], a["bt"], a["sl"], a["bs"], a["scale"], a["out"], a["B"],
             a["Hq"], a["Hkv"], a["d"], a["maxb"], a["NB"], a["maxL"], a["qdt"], a["kvdt"],
             a["odt"], a["ks"], a["vs"], a["P"], None)


def test_noalloc_decode_checks_arguments_before_its_scratch(lib):
    """Every argument error is reported as such, on the host, before the
    scratch array is looked up or cleared (no device is touched)."""
    assert _decode_noalloc(lib, Hq=6, Hkv=4) == 1
    assert _decode_noalloc(lib, d=96) == 2
    assert _decode_noalloc(lib, out=None) == 1
    assert _decode_noalloc(lib, kvdt=2) == 1     # fp8 cache without scales
    assert _decode_noalloc(lib, scale=float("inf")) == 1
    assert _decode_noalloc(lib, B=0) == 0        # empty batch: nothing to do


def test_internal_fault_setter_rejects_bad_modes(lib):
    """The test-only fault setter (exported, not in the public header) accepts
    only its known modes and a wait bound in (0, 2 s]."""
    f = lib.pkv_internal_decode_fault
    f.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_ulonglong]
    f.restype = ctypes.c_int
    assert f(7, 0, 1000000) == 1
    assert f(1, -1, 1000000) == 1
    assert f(1, 0, 0) == 1
    assert f(1, 0, 3_000_000_000) == 1
    assert f(0, 0, 1000000) == 0  # disarm
