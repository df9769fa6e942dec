"""B200 paged KV-cache library -- Python binding.

Argument marshalling only: every call goes straight to the C ABI in
``libpkv.so`` (declared in ``include/pkv.h``) with raw device pointers taken
from torch tensors and the current torch CUDA stream.  There is no CPU or
eager-torch fallback: the library is loaded on first use, and if it is not
built every call raises ImportError (build it with
``python -m paged_kv_cache_412_b200.build``).

Calls (names follow the C ABI):

* :func:`kv_cache_write` -- scatter new tokens' K/V into their cache slots.
* :func:`paged_attention_decode` -- one decode step of attention over the
  block-paged cache.
* :func:`copy_blocks` -- copy-on-write copy of physical blocks.
* :func:`decode_workspace_bytes`, :func:`get_device_error`.

Cache layout: ``[num_blocks, num_kv_heads, block_size, head_dim]``.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = [
    "PkvError", "LIB_PATH", "lib", "kv_cache_write", "paged_attention_decode", "copy_blocks",
    "decode_workspace_bytes", "new_workspace", "get_device_error", "status_string", "DEVERR",
    "paged_attention_decode_noalloc", "BlockAllocator", "waste_compare", "swap_blocks",
    "kv_cache_write_fp8", "workspace_init", "paged_attention_decode_append",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpkv.so")

PKV_OK = 0
STATUS_NAMES = {0: "PKV_OK", 1: "PKV_ERR_INVALID_ARG", 2: "PKV_ERR_UNSUPPORTED",
                3: "PKV_ERR_WORKSPACE", 4: "PKV_ERR_CUDA", 5: "PKV_ERR_DEVICE_INDEX"}
DEVERR = {"BAD_SLOT": 0x1, "BAD_BLOCK": 0x2, "BAD_SEQ_LEN": 0x4, "BAD_PAIR": 0x8,
          "TIMEOUT": 0x10, "PREFIX": 0x20}

_F32, _BF16, _FP8 = 0, 1, 2


class PkvError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is not built; run `python -m paged_kv_cache_412_b200.build` "
            "(the library has no fallback path)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                             ctypes.c_size_t)
    L.pkv_status_string.argtypes = [ctypes.c_int]
    L.pkv_status_string.restype = ctypes.c_char_p
    L.pkv_version.argtypes = []
    L.pkv_version.restype = ctypes.c_int
    L.pkv_kv_cache_write.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, ctypes.c_int, vp]
    L.pkv_kv_cache_write.restype = ctypes.c_int
    L.pkv_decode_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32, i32]
    L.pkv_decode_workspace_bytes.restype = sz
    L.pkv_decode_workspace_init.argtypes = [vp, sz, vp]
    L.pkv_decode_workspace_init.restype = ctypes.c_int
    L.pkv_paged_attention_decode.argtypes = [vp, vp, vp, vp, vp, i32, f32, vp, i32, i32, i32,
                                             i32, i32, i32, i32, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, vp, vp, i32, vp, sz, vp]
    L.pkv_paged_attention_decode.restype = ctypes.c_int
    L.pkv_paged_attention_decode_append.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, f32, vp,
                                                    i32, i32, i32, i32, i32, i32, i32,
                                                    ctypes.c_int, i32, vp, sz, vp]
    L.pkv_paged_attention_decode_append.restype = ctypes.c_int
    L.pkv_decode_prefix_workspace_bytes.argtypes = [i32] * 9
    L.pkv_decode_prefix_workspace_bytes.restype = sz
    L.pkv_paged_attention_decode_prefix.argtypes = [vp, vp, vp, vp, vp, i32, f32, vp, i32, i32,
                                                    i32, i32, i32, i32, i32, ctypes.c_int,
                                                    ctypes.c_int, ctypes.c_int, vp, vp, i32, i32,
                                                    i32, vp, sz, vp]
    L.pkv_paged_attention_decode_prefix.restype = ctypes.c_int
    L.pkv_copy_blocks.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, ctypes.c_int, vp]
    L.pkv_copy_blocks.restype = ctypes.c_int
    L.pkv_get_device_error.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
    L.pkv_get_device_error.restype = ctypes.c_int
    return L


_lib = None
_lib_lock = threading.Lock()


def _get_lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        with _lib_lock:
            if _lib is None:
                _lib = _load()
    return _lib


def __getattr__(name):
    if name == "lib":
        return _get_lib()
    raise AttributeError(name)


def status_string(status: int) -> str:
    return _get_lib().pkv_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != PKV_OK:
        raise PkvError(fn, status)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return _F32
    if t.dtype == torch.bfloat16:
        return _BF16
    if t.dtype in (torch.float8_e4m3fn, torch.uint8):
        return _FP8
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need_cuda(*ts: torch.Tensor) -> torch.device:
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")
        if not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("all tensors must be on one device")
    return dev


def kv_cache_write(k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor,
                   k_cache: torch.Tensor, v_cache: torch.Tensor) -> None:
    """k, v [T, Hkv, d]; slot_mapping [T] int64; caches [NB, Hkv, bs, d]."""
    dev = _need_cuda(k, v, slot_mapping, k_cache, v_cache)
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    if k.dtype != k_cache.dtype or v.dtype != v_cache.dtype or k.dtype != v.dtype:
        raise TypeError("k, v and the caches must share one dtype")
    T, Hkv, d = k.shape
    NB, Hkv2, bs, d2 = k_cache.shape
    if (Hkv, d) != (Hkv2, d2) or v.shape != k.shape or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    with torch.cuda.device(dev):
        st = _get_lib().pkv_kv_cache_write(_ptr(k), _ptr(v), _ptr(slot_mapping), _ptr(k_cache),
                                    _ptr(v_cache), T, Hkv, d, bs, NB, _dtype_code(k_cache),
                                    _stream(dev))
    _check("pkv_kv_cache_write", st)


def decode_workspace_bytes(num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                           block_size: int, max_seq_len: int, partition_size: int = 0) -> int:
    return int(_get_lib().pkv_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                              block_size, max_seq_len, partition_size))


_ws_lock = threading.Lock()
_ws_cache: dict = {}


def new_workspace(nbytes: int, device: torch.device | None = None) -> torch.Tensor:
    """Allocate (through torch) and initialise a decode workspace of nbytes."""
    dev = device or torch.device("cuda", torch.cuda.current_device())
    buf = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _check("pkv_decode_workspace_init",
               _get_lib().pkv_decode_workspace_init(_ptr(buf), buf.numel(), _stream(dev)))
    return buf


def workspace_init(workspace: torch.Tensor) -> None:
    """Zero a decode workspace on the current stream (pkv_decode_workspace_init):
    once after allocating it, and again after a call reported TIMEOUT."""
    dev = _need_cuda(workspace)
    with torch.cuda.device(dev):
        _check("pkv_decode_workspace_init",
               _get_lib().pkv_decode_workspace_init(
                   _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(dev)))


def _workspace(dev: torch.device, nbytes: int) -> torch.Tensor:
    """A per-(device, stream) scratch buffer, grown on demand (caller-side
    allocation through torch; the library itself allocates nothing)."""
    key = (dev.index, torch.cuda.current_stream(dev).cuda_stream)
    with _ws_lock:
        buf = _ws_cache.get(key)
        if buf is None or buf.numel() < nbytes:
            buf = new_workspace(nbytes, dev)
            _ws_cache[key] = buf
        return buf


def paged_attention_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                           block_tables: torch.Tensor, seq_lens: torch.Tensor,
                           block_size: int | None = None, scale: float | None = None,
                           out: torch.Tensor | None = None, *, max_seq_len: int | None = None,
                           partition_size: int = 0, out_dtype: torch.dtype | None = None,
                           k_scale: torch.Tensor | None = None,
                           v_scale: torch.Tensor | None = None,
                           workspace: torch.Tensor | None = None) -> torch.Tensor:
    """out[b, h] = softmax(scale * q[b, h] . K^T) V over request b's tokens.

    q [B, Hq, d]; caches [NB, Hkv, bs, d]; block_tables [B, max_blocks] int32;
    seq_lens [B] int32.  ``max_seq_len`` defaults to the block tables' capacity.
    """
    dev = _need_cuda(q, k_cache, v_cache, block_tables, seq_lens, out, k_scale, v_scale,
                     workspace)
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("block_tables and seq_lens must be int32")
    B, Hq, d = q.shape
    NB, Hkv, bs, d2 = k_cache.shape
    if block_size is None:
        block_size = bs
    if block_size != bs or d2 != d or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    if scale is None:
        scale = d ** -0.5
    max_blocks = block_tables.shape[1]
    if max_seq_len is None:
        max_seq_len = max_blocks * bs
    if out is None:
        out = torch.empty((B, Hq, d), dtype=out_dtype or q.dtype, device=dev)
    with torch.cuda.device(dev):
        # a caller's workspace is checked by the library itself
        ws = workspace if workspace is not None else _workspace(
            dev, decode_workspace_bytes(B, Hq, Hkv, d, bs, max_seq_len, partition_size))
        st = _get_lib().pkv_paged_attention_decode(
            _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(seq_lens),
            bs, float(scale), _ptr(out), B, Hq, Hkv, d, max_blocks, NB, int(max_seq_len),
            _dtype_code(q), _dtype_code(k_cache), _dtype_code(out), _ptr(k_scale),
            _ptr(v_scale), int(partition_size), _ptr(ws), ws.numel() * ws.element_size(),
            _stream(dev))
    _check("pkv_paged_attention_decode", st)
    return out


def paged_attention_decode_append(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                                  k_cache: torch.Tensor, v_cache: torch.Tensor,
                                  block_tables: torch.Tensor, seq_lens: torch.Tensor,
                                  block_size: int | None = None, scale: float | None = None,
                                  out: torch.Tensor | None = None, *,
                                  max_seq_len: int | None = None, partition_size: int = 0,
                                  out_dtype: torch.dtype | None = None,
                                  workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Append each request's new token, then paged_attention_decode.

    k_new, v_new [B, Hkv, d] bf16: the K and V rows of request b's token at
    position seq_lens[b] - 1, written to the slot its block table names (the
    bytes kv_cache_write writes there) before the decode reads that block --
    inside the decode launch when the decode runs one CTA per SM, else by a
    small kernel launched first.  bf16 q and caches, head_dim 64 or 128,
    block_size >= 2.
    """
    dev = _need_cuda(q, k_new, v_new, k_cache, v_cache, block_tables, seq_lens, out, workspace)
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("block_tables and seq_lens must be int32")
    for name, t in (("q", q), ("k_new", k_new), ("v_new", v_new), ("k_cache", k_cache),
                    ("v_cache", v_cache)):
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16")
    B, Hq, d = q.shape
    NB, Hkv, bs, d2 = k_cache.shape
    if block_size is None:
        block_size = bs
    if (block_size != bs or d2 != d or v_cache.shape != k_cache.shape
            or tuple(k_new.shape) != (B, Hkv, d) or v_new.shape != k_new.shape):
        raise ValueError("shape mismatch")
    if scale is None:
        scale = d ** -0.5
    max_blocks = block_tables.shape[1]
    if max_seq_len is None:
        max_seq_len = max_blocks * bs
    if out is None:
        out = torch.empty((B, Hq, d), dtype=out_dtype or q.dtype, device=dev)
    with torch.cuda.device(dev):
        ws = workspace if workspace is not None else _workspace(
            dev, decode_workspace_bytes(B, Hq, Hkv, d, bs, max_seq_len, partition_size))
        st = _get_lib().pkv_paged_attention_decode_append(
            _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
            _ptr(seq_lens), bs, float(scale), _ptr(out), B, Hq, Hkv, d, max_blocks, NB,
            int(max_seq_len), _dtype_code(out), int(partition_size), _ptr(ws),
            ws.numel() * ws.element_size(), _stream(dev))
    _check("pkv_paged_attention_decode_append", st)
    return out


def decode_prefix_workspace_bytes(num_seqs: int, num_q_heads: int, num_kv_heads: int,
                                  head_dim: int, block_size: int, max_seq_len: int,
                                  num_prefixes: int, max_prefix_members: int,
                                  max_prefix_len: int) -> int:
    return int(_get_lib().pkv_decode_prefix_workspace_bytes(
        num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_seq_len, num_prefixes,
        max_prefix_members, max_prefix_len))


def paged_attention_decode_prefix(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                                  block_tables: torch.Tensor, seq_lens: torch.Tensor,
                                  prefix_of: torch.Tensor, prefix_lens: torch.Tensor,
                                  block_size: int | None = None, scale: float | None = None,
                                  out: torch.Tensor | None = None, *,
                                  max_seq_len: int | None = None,
                                  max_prefix_members: int | None = None,
                                  max_prefix_len: int | None = None,
                                  out_dtype: torch.dtype | None = None,
                                  workspace: torch.Tensor | None = None) -> torch.Tensor:
    """paged_attention_decode for requests that share prefix blocks.

    prefix_of [B] int32: the group of each request (-1: none); prefix_lens [G]
    int32: tokens of each group's shared prefix (a multiple of block_size).
    The group's shared blocks are read once for all its members, then each
    request's own tokens; the result equals paged_attention_decode.
    ``max_prefix_members`` defaults to B and ``max_prefix_len`` to max_seq_len.
    """
    dev = _need_cuda(q, k_cache, v_cache, block_tables, seq_lens, prefix_of, prefix_lens, out,
                     workspace)
    for name, t in (("block_tables", block_tables), ("seq_lens", seq_lens),
                    ("prefix_of", prefix_of), ("prefix_lens", prefix_lens)):
        if t.dtype != torch.int32:
            raise TypeError(f"{name} must be int32")
    B, Hq, d = q.shape
    NB, Hkv, bs, d2 = k_cache.shape
    if block_size is None:
        block_size = bs
    if block_size != bs or d2 != d or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    if prefix_of.numel() != B:
        raise ValueError("prefix_of must hold one entry per request")
    if scale is None:
        scale = d ** -0.5
    max_blocks = block_tables.shape[1]
    if max_seq_len is None:
        max_seq_len = max_blocks * bs
    if max_prefix_members is None:
        max_prefix_members = max(B, 1)
    if max_prefix_len is None:
        max_prefix_len = max_seq_len
    G = prefix_lens.numel()
    if out is None:
        out = torch.empty((B, Hq, d), dtype=out_dtype or q.dtype, device=dev)
    need = decode_prefix_workspace_bytes(B, Hq, Hkv, d, bs, max_seq_len, G, max_prefix_members,
                                         max_prefix_len)
    if need == 0:
        raise PkvError("pkv_decode_prefix_workspace_bytes", 1)
    with torch.cuda.device(dev):
        ws = workspace if workspace is not None else _workspace(dev, need)
        st = _get_lib().pkv_paged_attention_decode_prefix(
            _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(seq_lens), bs,
            float(scale), _ptr(out), B, Hq, Hkv, d, max_blocks, NB, int(max_seq_len),
            _dtype_code(q), _dtype_code(k_cache), _dtype_code(out), _ptr(prefix_of),
            _ptr(prefix_lens), G, int(max_prefix_members), int(max_prefix_len), _ptr(ws),
            ws.numel() * ws.element_size(), _stream(dev))
    _check("pkv_paged_attention_decode_prefix", st)
    return out


_fp8w_declared = False


def kv_cache_write_fp8(k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor,
                       k_cache: torch.Tensor, v_cache: torch.Tensor, k_scale: torch.Tensor,
                       v_scale: torch.Tensor) -> None:
    """Quantising append: k, v [T, Hkv, d] bf16 -> e4m3 codes (uint8 caches
    [NB, Hkv, bs, d]) of x / scale[h]; k_scale, v_scale [Hkv] fp32 on device."""
    global _fp8w_declared
    L = _get_lib()
    if not _fp8w_declared:
        vp, i32 = ctypes.c_void_p, ctypes.c_int32
        L.pkv_kv_cache_write_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                             vp]
        L.pkv_kv_cache_write_fp8.restype = ctypes.c_int
        _fp8w_declared = True
    dev = _need_cuda(k, v, slot_mapping, k_cache, v_cache, k_scale, v_scale)
    if k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
        raise TypeError("k and v must be bf16")
    if k_cache.dtype not in (torch.uint8, torch.float8_e4m3fn) or v_cache.dtype != k_cache.dtype:
        raise TypeError("fp8 caches must be uint8 or float8_e4m3fn")
    if k_scale.dtype != torch.float32 or v_scale.dtype != torch.float32:
        raise TypeError("scales must be float32")
    T, Hkv, d = k.shape
    NB, _, bs, _ = k_cache.shape
    with torch.cuda.device(dev):
        st = L.pkv_kv_cache_write_fp8(_ptr(k), _ptr(v), _ptr(slot_mapping), _ptr(k_cache),
                                      _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), T, Hkv, d, bs,
                                      NB, _stream(dev))
    _check("pkv_kv_cache_write_fp8", st)


_swap_declared = False


def swap_blocks(src_k: torch.Tensor, src_v: torch.Tensor, dst_k: torch.Tensor,
                dst_v: torch.Tensor, block_mapping: torch.Tensor,
                device: torch.device | int | None = None) -> None:
    """dst pools[dst] = src pools[src] for each (src, dst) row of block_mapping.

    Pools are [num_blocks, Hkv, bs, d]; each may be a CUDA tensor or a pinned
    CPU tensor (``pin_memory()``); block_mapping likewise.  The copy runs on the
    current stream of ``device`` (default: the CUDA tensor's device, else the
    current device)."""
    global _swap_declared
    L = _get_lib()
    if not _swap_declared:
        vp, i32 = ctypes.c_void_p, ctypes.c_int32
        L.pkv_swap_blocks.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                      ctypes.c_int, vp]
        L.pkv_swap_blocks.restype = ctypes.c_int
        _swap_declared = True
    ts = (src_k, src_v, dst_k, dst_v, block_mapping)
    for t in ts:
        if not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")
        if not t.is_cuda and not t.is_pinned():
            raise ValueError("CPU tensors must be pinned (pin_memory())")
    if device is None:
        cuda = [t.device for t in ts if t.is_cuda]
        device = cuda[0] if cuda else torch.device("cuda", torch.cuda.current_device())
    dev = torch.device("cuda", device) if isinstance(device, int) else device
    if block_mapping.dtype != torch.int64:
        raise TypeError("block_mapping must be int64")
    if src_k.dtype != dst_k.dtype or src_k.shape[1:] != dst_k.shape[1:]:
        raise ValueError("pools must share dtype and block shape")
    n = block_mapping.numel() // 2
    NBs, Hkv, bs, d = src_k.shape
    with torch.cuda.device(dev):
        st = L.pkv_swap_blocks(_ptr(src_k), _ptr(src_v), _ptr(dst_k), _ptr(dst_v),
                               _ptr(block_mapping), n, NBs, dst_k.shape[0], Hkv, d, bs,
                               _dtype_code(src_k), _stream(dev))
    _check("pkv_swap_blocks", st)


_noalloc_declared = False


def paged_attention_decode_noalloc(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                                   block_tables: torch.Tensor, seq_lens: torch.Tensor,
                                   block_size: int | None = None, scale: float | None = None,
                                   out: torch.Tensor | None = None, *,
                                   max_seq_len: int | None = None, partition_size: int = 0,
                                   out_dtype: torch.dtype | None = None,
                                   k_scale: torch.Tensor | None = None,
                                   v_scale: torch.Tensor | None = None) -> torch.Tensor:
    """The same decode through ``pkv_paged_attention_decode_noalloc``: no
    workspace argument, the library's fixed device scratch array is used.

    For callers that may not allocate device memory (see the C header).  Calls
    on one device share that array and must not overlap on the GPU.
    ``k_scale`` / ``v_scale`` as in :func:`paged_attention_decode` (fp8 caches).
    """
    global _noalloc_declared
    L = _get_lib()
    if not _noalloc_declared:
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        L.pkv_paged_attention_decode_noalloc.argtypes = [
            vp, vp, vp, vp, vp, i32, ctypes.c_float, vp, i32, i32, i32, i32, i32, i32, i32,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, i32, vp]
        L.pkv_paged_attention_decode_noalloc.restype = ctypes.c_int
        L.pkv_decode_noalloc_scratch_bytes.argtypes = []
        L.pkv_decode_noalloc_scratch_bytes.restype = sz
        _noalloc_declared = True
    dev = _need_cuda(q, k_cache, v_cache, block_tables, seq_lens, out, k_scale, v_scale)
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("block_tables and seq_lens must be int32")
    B, Hq, d = q.shape
    NB, Hkv, bs, d2 = k_cache.shape
    if block_size is None:
        block_size = bs
    if block_size != bs or d2 != d or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    if scale is None:
        scale = d ** -0.5
    max_blocks = block_tables.shape[1]
    if max_seq_len is None:
        max_seq_len = max_blocks * bs
    if out is None:
        out = torch.empty((B, Hq, d), dtype=out_dtype or q.dtype, device=dev)
    with torch.cuda.device(dev):
        st = L.pkv_paged_attention_decode_noalloc(
            _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(seq_lens), bs,
            float(scale), _ptr(out), B, Hq, Hkv, d, max_blocks, NB, int(max_seq_len),
            _dtype_code(q), _dtype_code(k_cache), _dtype_code(out), _ptr(k_scale),
            _ptr(v_scale), int(partition_size), _stream(dev))
    _check("pkv_paged_attention_decode_noalloc", st)
    return out


def copy_blocks(k_cache: torch.Tensor, v_cache: torch.Tensor, block_mapping: torch.Tensor) -> None:
    """block_mapping [n, 2] int64 (src, dst): cache[dst] = cache[src] for K and V."""
    dev = _need_cuda(k_cache, v_cache, block_mapping)
    if block_mapping.dtype != torch.int64:
        raise TypeError("block_mapping must be int64")
    n = block_mapping.numel() // 2
    NB, Hkv, bs, d = k_cache.shape
    with torch.cuda.device(dev):
        st = _get_lib().pkv_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(block_mapping), n, Hkv, d,
                                 bs, NB, _dtype_code(k_cache), _stream(dev))
    _check("pkv_copy_blocks", st)


def get_device_error(device: torch.device | int | None = None) -> int:
    """Synchronise the current stream, then read and clear the device error
    word (PKV_DEVERR_* bits, see ``DEVERR``)."""
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else
                       (device if isinstance(device, int) else device.index))
    flags = ctypes.c_uint32(0)
    with torch.cuda.device(dev):
        st = _get_lib().pkv_get_device_error(_stream(dev), ctypes.byref(flags))
    if st not in (PKV_OK, 5):
        raise PkvError("pkv_get_device_error", st)
    return int(flags.value)


# ---------------------------------------------------------------------------
# host-side block manager (C++ in libpkv.so; no GPU work)
# ---------------------------------------------------------------------------

class _AllocStats(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("free_blocks", ctypes.c_int32),
                ("used_blocks", ctypes.c_int32), ("shared_blocks", ctypes.c_int32),
                ("num_seqs", ctypes.c_int32), ("stored_tokens", ctypes.c_int64),
                ("logical_tokens", ctypes.c_int64), ("unused_slots", ctypes.c_int64)]


class _WasteReport(ctypes.Structure):
    _fields_ = [("used_slots", ctypes.c_int64), ("contiguous_reserved", ctypes.c_int64),
                ("paged_reserved", ctypes.c_int64), ("contiguous_admitted", ctypes.c_int32),
                ("paged_admitted", ctypes.c_int32)]


_alloc_declared = False


def _alloc_lib():
    global _alloc_declared
    L = _get_lib()
    if not _alloc_declared:
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        P = ctypes.POINTER
        L.pkv_allocator_create.argtypes = [i32, i32, P(vp)]
        L.pkv_allocator_destroy.argtypes = [vp]
        L.pkv_allocator_destroy.restype = None
        L.pkv_allocator_add_seq.argtypes = [vp, i64]
        L.pkv_allocator_fork.argtypes = [vp, i64, i64]
        L.pkv_allocator_append.argtypes = [vp, i64, i32, P(i64), P(i64), P(i32)]
        L.pkv_allocator_free_seq.argtypes = [vp, i64]
        L.pkv_allocator_block_table.argtypes = [vp, i64, P(i32), i32, P(i32), P(i64)]
        L.pkv_allocator_get_stats.argtypes = [vp, P(_AllocStats)]
        L.pkv_allocator_refcount.argtypes = [vp, i32]
        L.pkv_allocator_refcount.restype = i32
        L.pkv_waste_compare.argtypes = [P(i32), i32, i32, i32, i64, P(_WasteReport)]
        for f in ("pkv_allocator_create", "pkv_allocator_add_seq", "pkv_allocator_fork",
                  "pkv_allocator_append", "pkv_allocator_free_seq", "pkv_allocator_block_table",
                  "pkv_allocator_get_stats", "pkv_waste_compare"):
            getattr(L, f).restype = ctypes.c_int
        _alloc_declared = True
    return L


class BlockAllocator:
    """Physical-block pool with per-sequence block tables, reference-counted
    sharing (fork) and copy-on-write on append.  Host memory only."""

    def __init__(self, num_blocks: int, block_size: int):
        import numpy as np  # noqa: F401  (numpy arrays are returned)
        self._L = _alloc_lib()
        h = ctypes.c_void_p()
        _check("pkv_allocator_create", self._L.pkv_allocator_create(num_blocks, block_size,
                                                                    ctypes.byref(h)))
        self._h = h
        self.num_blocks, self.block_size = num_blocks, block_size

    def close(self) -> None:
        if getattr(self, "_h", None):
            self._L.pkv_allocator_destroy(self._h)
            self._h = None

    __del__ = close

    def add_seq(self, seq_id: int) -> None:
        _check("pkv_allocator_add_seq", self._L.pkv_allocator_add_seq(self._h, seq_id))

    def fork(self, parent: int, child: int) -> None:
        _check("pkv_allocator_fork", self._L.pkv_allocator_fork(self._h, parent, child))

    def append(self, seq_id: int, num_tokens: int):
        """Returns (slots int64[num_tokens], copy-on-write pair (src, dst) or None)."""
        import numpy as np
        slots = np.zeros(max(num_tokens, 1), dtype=np.int64)
        pair = (ctypes.c_int64 * 2)()
        ncow = ctypes.c_int32(0)
        st = self._L.pkv_allocator_append(self._h, seq_id, num_tokens,
                                          slots.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                          pair, ctypes.byref(ncow))
        _check("pkv_allocator_append", st)
        return slots[:num_tokens], ((int(pair[0]), int(pair[1])) if ncow.value else None)

    def free_seq(self, seq_id: int) -> None:
        _check("pkv_allocator_free_seq", self._L.pkv_allocator_free_seq(self._h, seq_id))

    def block_table(self, seq_id: int):
        """Returns (int32 block ids, number of tokens)."""
        import numpy as np
        nb, nt = ctypes.c_int32(0), ctypes.c_int64(0)
        self._L.pkv_allocator_block_table(self._h, seq_id, None, 0, ctypes.byref(nb),
                                          ctypes.byref(nt))
        table = np.zeros(max(nb.value, 1), dtype=np.int32)
        _check("pkv_allocator_block_table", self._L.pkv_allocator_block_table(
            self._h, seq_id, table.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), table.size,
            ctypes.byref(nb), ctypes.byref(nt)))
        return table[:nb.value], int(nt.value)

    def stats(self) -> dict:
        s = _AllocStats()
        _check("pkv_allocator_get_stats", self._L.pkv_allocator_get_stats(self._h,
                                                                          ctypes.byref(s)))
        return {k: getattr(s, k) for k, _ in _AllocStats._fields_}

    def refcount(self, block: int) -> int:
        return int(self._L.pkv_allocator_refcount(self._h, block))


def waste_compare(lengths, reserve_len: int, block_size: int, pool_slots: int) -> dict:
    """Contiguous (reserve_len per request) vs paged (whole blocks) reservation:
    slots used/reserved and how many requests fit at once in pool_slots."""
    import numpy as np
    L = _alloc_lib()
    arr = np.ascontiguousarray(lengths, dtype=np.int32)
    r = _WasteReport()
    _check("pkv_waste_compare", L.pkv_waste_compare(
        arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), arr.size, reserve_len, block_size,
        pool_slots, ctypes.byref(r)))
    return {k: getattr(r, k) for k, _ in _WasteReport._fields_}
