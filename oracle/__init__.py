"""CPU oracle for the paged KV-cache hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never calls it and
shares no code with it; the only thing both sides consume is the seeded input
generator in ``workloads.py``, which holds none of the method's arithmetic.

The arithmetic lives in ``pkv_oracle.c`` (plain C, fp64, OpenMP over
independent (request, query head) pairs).  This module compiles it with gcc on
first use (or via :func:`build`) and wraps each entry point for numpy arrays.

Functions and the passages they follow (page title, section):

* :func:`decode` -- paged decode attention, plain definition: gather each
  request's blocks through its block table into contiguous fp64 K/V, then
  ``softmax(q K^T * scale) V``.  "PagedAttention: Optimizing KV Cache
  Utilization in Large Language Models", "The Mechanics of PagedAttention" and
  "The Math: Block Attention Calculation"; "KV Cache Management", "The
  Solution: PagedAttention (vLLM)".
* :func:`decode_weights` -- the softmax weights of one (request, head) pair.
* :func:`decode_partitioned` -- split-sequence restatement (per-block running
  max / normaliser, per-partition partials, merge), pinned against
  :func:`decode`.
* :func:`kv_cache_write` -- scatter of new tokens' K/V into their slots
  ("The Mechanics of PagedAttention": vectors written into scattered blocks).
* :func:`copy_blocks` -- copy-on-write copy of whole physical blocks ("KV Cache
  Optimization and PagedAttention", intro on shared prefix blocks; "KV Cache
  Management", "The Bonus: Zero-Copy Sharing").
* :func:`swap_blocks` -- block copy between two pools (preemption swap;
  "PagedAttention: Optimizing ...", "Conclusion").

Pins: every function is checked in ``tests/test_oracle.py`` against things the
pages and mathematics fix (brute force, permutation and block-size invariance,
shared-prefix equality, closed forms, planted mistakes).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pkv_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")

F32, BF16, FP8E4M3 = 0, 1, 2

_lock = threading.Lock()
_lib = None


def build(mutant: int = 0, out_path: str | None = None) -> str:
    """Compile the oracle with gcc.  ``mutant`` != 0 plants one numbered mistake
    (used only by the oracle's self-test); the product oracle is mutant 0."""
    path = out_path or _LIB_PATH
    os.makedirs(os.path.dirname(path), exist_ok=True)
    cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
           f"-DORACLE_MUTANT={int(mutant)}", "-o", path, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return path


def _declare(lib):
    vp, i32p, i64p, f32p, f64p = (ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32),
                                  ctypes.POINTER(ctypes.c_int64),
                                  ctypes.POINTER(ctypes.c_float),
                                  ctypes.POINTER(ctypes.c_double))
    ci, cd = ctypes.c_int, ctypes.c_double
    lib.oracle_decode.argtypes = [vp, ci, vp, vp, ci, f32p, f32p, i32p, i32p, ci, ci,
                                  ci, ci, ci, ci, ci, cd, f64p, ci]
    lib.oracle_decode.restype = ci
    lib.oracle_decode_weights.argtypes = [vp, ci, vp, vp, ci, f32p, f32p, i32p, i32p,
                                          ci, ci, ci, ci, ci, ci, cd, ci, ci, f64p]
    lib.oracle_decode_weights.restype = ci
    lib.oracle_decode_partitioned.argtypes = [vp, ci, vp, vp, ci, f32p, f32p, i32p,
                                              i32p, ci, ci, ci, ci, ci, ci, ci, cd,
                                              ci, f64p]
    lib.oracle_decode_partitioned.restype = ci
    lib.oracle_kv_cache_write.argtypes = [vp, vp, i64p, vp, vp, ci, ci, ci, ci, ci, ci]
    lib.oracle_kv_cache_write.restype = ci
    lib.oracle_copy_blocks.argtypes = [vp, vp, i64p, ci, ci, ci, ci, ci, ci]
    lib.oracle_copy_blocks.restype = ci
    lib.oracle_swap_blocks.argtypes = [vp, vp, vp, vp, i64p, ci, ci, ci, ci, ci, ci, ci]
    lib.oracle_swap_blocks.restype = ci
    lib.oracle_max_threads.argtypes = []
    lib.oracle_max_threads.restype = ci
    lib.oracle_quantize_e4m3.argtypes = [f32p, ci, ctypes.c_float,
                                         ctypes.POINTER(ctypes.c_uint8)]
    lib.oracle_quantize_e4m3.restype = None
    return lib


def load(path: str | None = None):
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            stale = (not os.path.exists(_LIB_PATH) or
                     os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
            if stale:
                build()
            _lib = _declare(ctypes.CDLL(_LIB_PATH))
    return _lib


# --------------------------------------------------------------------------
# numpy wrappers
# --------------------------------------------------------------------------

def _dtype_code(arr: np.ndarray, fp8: bool = False) -> int:
    if arr.dtype == np.float32:
        return F32
    if arr.dtype == np.uint16:  # bf16 bit patterns
        return BF16
    if arr.dtype == np.uint8 and fp8:
        return FP8E4M3
    raise TypeError(f"oracle: unsupported element array dtype {arr.dtype}")


def _ptr(a, ctype=None):
    if a is None:
        return None
    if ctype is None:
        return ctypes.c_void_p(a.ctypes.data)
    return a.ctypes.data_as(ctypes.POINTER(ctype))


class OracleError(RuntimeError):
    pass


def decode(q, k_cache, v_cache, block_tables, seq_lens, scale, *, k_scale=None,
           v_scale=None, nthreads: int = 0, lib=None) -> np.ndarray:
    """Plain paged decode attention in fp64.

    q [B, Hq, d] (float32 or bf16 bits as uint16); k_cache / v_cache
    [NB, Hkv, bs, d] (float32, bf16 bits, or fp8 e4m3 bits as uint8 with
    per-kv-head ``k_scale`` / ``v_scale``); block_tables [B, max_blocks] int32;
    seq_lens [B] int32.  Returns out [B, Hq, d] float64.
    """
    lib = lib or load()
    q = np.ascontiguousarray(q)
    k_cache = np.ascontiguousarray(k_cache)
    v_cache = np.ascontiguousarray(v_cache)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, Hq, d = q.shape
    NB, Hkv, bs, d2 = k_cache.shape
    assert d2 == d and v_cache.shape == k_cache.shape
    fp8 = k_scale is not None
    ks = None if k_scale is None else np.ascontiguousarray(k_scale, dtype=np.float32)
    vs = None if v_scale is None else np.ascontiguousarray(v_scale, dtype=np.float32)
    out = np.zeros((B, Hq, d), dtype=np.float64)
    st = lib.oracle_decode(_ptr(q), _dtype_code(q), _ptr(k_cache), _ptr(v_cache),
                           _dtype_code(k_cache, fp8), _ptr(ks, ctypes.c_float),
                           _ptr(vs, ctypes.c_float), _ptr(bt, ctypes.c_int32),
                           _ptr(sl, ctypes.c_int32), B, Hq, Hkv, d, bs,
                           bt.shape[1] if bt.ndim == 2 else 0, NB, float(scale),
                           _ptr(out, ctypes.c_double), int(nthreads))
    if st != 0:
        raise OracleError(f"oracle_decode failed with status {st}")
    return out


def decode_weights(q, k_cache, v_cache, block_tables, seq_lens, scale, b, h, *,
                   k_scale=None, v_scale=None, lib=None) -> np.ndarray:
    """Softmax weights (length seq_lens[b]) of request b, query head h."""
    lib = lib or load()
    q = np.ascontiguousarray(q)
    k_cache = np.ascontiguousarray(k_cache)
    v_cache = np.ascontiguousarray(v_cache)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, Hq, d = q.shape
    NB, Hkv, bs, _ = k_cache.shape
    fp8 = k_scale is not None
    ks = None if k_scale is None else np.ascontiguousarray(k_scale, dtype=np.float32)
    vs = None if v_scale is None else np.ascontiguousarray(v_scale, dtype=np.float32)
    w = np.zeros(max(int(sl[b]), 1), dtype=np.float64)
    st = lib.oracle_decode_weights(_ptr(q), _dtype_code(q), _ptr(k_cache),
                                   _ptr(v_cache), _dtype_code(k_cache, fp8),
                                   _ptr(ks, ctypes.c_float), _ptr(vs, ctypes.c_float),
                                   _ptr(bt, ctypes.c_int32), _ptr(sl, ctypes.c_int32),
                                   Hq, Hkv, d, bs, bt.shape[1], NB, float(scale),
                                   int(b), int(h), _ptr(w, ctypes.c_double))
    if st != 0:
        raise OracleError(f"oracle_decode_weights failed with status {st}")
    return w[: int(sl[b])]


def decode_partitioned(q, k_cache, v_cache, block_tables, seq_lens, scale,
                       partition_tokens, *, k_scale=None, v_scale=None,
                       lib=None) -> np.ndarray:
    """Split-sequence restatement (partitions of ``partition_tokens``)."""
    lib = lib or load()
    q = np.ascontiguousarray(q)
    k_cache = np.ascontiguousarray(k_cache)
    v_cache = np.ascontiguousarray(v_cache)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, Hq, d = q.shape
    NB, Hkv, bs, _ = k_cache.shape
    fp8 = k_scale is not None
    ks = None if k_scale is None else np.ascontiguousarray(k_scale, dtype=np.float32)
    vs = None if v_scale is None else np.ascontiguousarray(v_scale, dtype=np.float32)
    out = np.zeros((B, Hq, d), dtype=np.float64)
    st = lib.oracle_decode_partitioned(_ptr(q), _dtype_code(q), _ptr(k_cache),
                                       _ptr(v_cache), _dtype_code(k_cache, fp8),
                                       _ptr(ks, ctypes.c_float),
                                       _ptr(vs, ctypes.c_float),
                                       _ptr(bt, ctypes.c_int32),
                                       _ptr(sl, ctypes.c_int32), B, Hq, Hkv, d, bs,
                                       bt.shape[1], NB, float(scale),
                                       int(partition_tokens),
                                       _ptr(out, ctypes.c_double))
    if st != 0:
        raise OracleError(f"oracle_decode_partitioned failed with status {st}")
    return out


def kv_cache_write(k, v, slot_mapping, k_cache, v_cache, *, lib=None) -> int:
    """In-place scatter of k/v [T, Hkv, d] into the caches [NB, Hkv, bs, d].
    Returns the number of tokens skipped for an out-of-range slot."""
    lib = lib or load()
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    assert k.dtype == k_cache.dtype == v.dtype == v_cache.dtype
    T, Hkv, d = k.shape
    NB, Hkv2, bs, d2 = k_cache.shape
    assert Hkv == Hkv2 and d == d2
    return lib.oracle_kv_cache_write(_ptr(k), _ptr(v), _ptr(sm, ctypes.c_int64),
                                     _ptr(k_cache), _ptr(v_cache), T, NB, Hkv, d, bs,
                                     k.dtype.itemsize)


def copy_blocks(k_cache, v_cache, block_mapping, *, lib=None) -> int:
    """In-place cache[dst] = cache[src] for each (src, dst) row of block_mapping."""
    lib = lib or load()
    bm = np.ascontiguousarray(block_mapping, dtype=np.int64).reshape(-1, 2)
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    NB, Hkv, bs, d = k_cache.shape
    return lib.oracle_copy_blocks(_ptr(k_cache), _ptr(v_cache),
                                  _ptr(bm, ctypes.c_int64), bm.shape[0], NB, Hkv, d,
                                  bs, k_cache.dtype.itemsize)


def swap_blocks(src_k, src_v, dst_k, dst_v, block_mapping, *, lib=None) -> int:
    """dst pools[dst] = src pools[src] for each (src, dst) row of block_mapping."""
    lib = lib or load()
    bm = np.ascontiguousarray(block_mapping, dtype=np.int64).reshape(-1, 2)
    NBs, Hkv, bs, d = src_k.shape
    NBd = dst_k.shape[0]
    return lib.oracle_swap_blocks(_ptr(src_k), _ptr(src_v), _ptr(dst_k), _ptr(dst_v),
                                  _ptr(bm, ctypes.c_int64), bm.shape[0], NBs, NBd,
                                  Hkv, d, bs, src_k.dtype.itemsize)


def quantize_e4m3(x: np.ndarray, scale: float, *, lib=None) -> np.ndarray:
    """fp8 e4m3 codes of x / scale (fp32 quotient, round to nearest even,
    saturating at +-448)."""
    lib = lib or load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.zeros(x.shape, dtype=np.uint8)
    lib.oracle_quantize_e4m3(_ptr(x, ctypes.c_float), x.size, ctypes.c_float(scale),
                             _ptr(out, ctypes.c_uint8))
    return out


def max_threads(lib=None) -> int:
    lib = lib or load()
    return lib.oracle_max_threads()
