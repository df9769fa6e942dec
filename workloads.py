"""Seeded synthetic inputs for the paged KV-cache hot path.

This module is the ONE thing the oracle side and the CUDA side both consume.
It holds none of the method's arithmetic: it draws random numbers, lays them
into the cache layout, builds block tables / slot mappings / copy pairs, and
nothing else.  All arrays are host numpy arrays.

Cache layout (a convention of this library; the pages do not fix one):
``k_cache`` / ``v_cache`` are ``[num_blocks, num_kv_heads, block_size, head_dim]``;
the token at logical position t of request b lives in physical block
``block_tables[b][t // block_size]`` at offset ``t % block_size``; a slot id is
``physical_block * block_size + offset``.

Workloads (shapes from the pages' examples: 32 q / 8 KV heads, head_dim 128,
block size 16, 4k-token requests, 128k contexts, a shared system prompt):

* ``tiny_f32``   batch 4, seq_lens [1, 17, 100, 200], 4 q / 2 KV heads, d 64,
  block 16, pool 64 blocks drawn by a seeded permutation, fp32.
* ``gqa_4k``     batch 16 x 4096 tokens, 32 q / 8 KV heads, d 128, block 16,
  4096 blocks randomly permuted, bf16.
* ``mixed``      256 requests, lengths log-uniform in [16, 8192], pool 1.1x
  the blocks needed, shuffled, bf16.
* ``prefix``     64 requests sharing a 2040-token prefix in 128 blocks (the
  last one partially filled and forked per request before appending), each
  with a 64..512-token suffix, bf16.
* ``long_ctx``   batch 2 x 131072 tokens, 64 q / 8 KV heads, block size 8,
  16 or 32, bf16.

Values: q, K, V ~ N(0, 1) in fp32 (numpy ``default_rng(seed)``), cast to bf16
with round-to-nearest-even where the workload is bf16; bf16 arrays are carried
as their uint16 bit patterns.  Cache slots no request owns (and the slots the
step's new tokens will fill) are NaN when ``poison=True`` (parity runs, so a
stray read or write shows up) and 0 otherwise (timed runs).
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

BF16_NAN = np.uint16(0x7FC0)
E4M3_NAN = np.uint8(0x7F)


_CHUNK = 1 << 22  # values per chunk of the threaded fills below
_THREADS = max(1, min(16, os.cpu_count() or 1))


def _chunked(n: int, fn) -> None:
    """Run fn(lo, hi) over [0, n) in chunks of _CHUNK on a thread pool (the
    numpy kernels used release the GIL); deterministic whatever the pool size."""
    spans = [(lo, min(lo + _CHUNK, n)) for lo in range(0, n, _CHUNK)]
    if len(spans) <= 1:
        for lo, hi in spans:
            fn(lo, hi)
        return
    with ThreadPoolExecutor(_THREADS) as ex:
        list(ex.map(lambda sp: fn(*sp), spans))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16, returned as uint16 bit patterns
    (finite inputs; 32-bit integer arithmetic cannot overflow for them)."""
    u = np.ascontiguousarray(x, dtype=np.float32).reshape(-1).view(np.uint32)
    out = np.empty(u.shape, dtype=np.uint16)

    def conv(lo, hi):
        v = u[lo:hi]
        r = (v >> 16) & 1
        r += 0x7FFF
        r += v
        r >>= 16
        out[lo:hi] = r

    _chunked(u.size, conv)
    return out.reshape(np.shape(x))


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    bs: int
    num_blocks: int
    dtype: str                      # "f32" or "bf16" (element type of q, K, V)
    scale: float
    q: np.ndarray                   # [B, Hq, d]
    k_cache: np.ndarray             # [NB, Hkv, bs, d] -- state BEFORE the step
    v_cache: np.ndarray
    block_tables: np.ndarray        # [B, max_blocks] int32, tail = -1
    seq_lens: np.ndarray            # [B] int32, lengths AFTER the step's append
    k_new: np.ndarray               # [T, Hkv, d] tokens the step appends
    v_new: np.ndarray
    slot_mapping: np.ndarray        # [T] int64
    copy_pairs: np.ndarray = field(default_factory=lambda: np.zeros((0, 2), np.int64))
    info: dict = field(default_factory=dict)
    k_scale: np.ndarray | None = None  # [Hkv] fp32, fp8 caches only
    v_scale: np.ndarray | None = None

    @property
    def max_blocks(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def elem_bytes(self) -> int:
        return {"f32": 4, "bf16": 2, "fp8": 1}[self.dtype]


def _normal(rng: np.random.Generator, shape, dtype: str) -> np.ndarray:
    """N(0, 1) fp32 values (bf16 bit patterns for bf16).  Chunk i of the
    flattened array is drawn from its own generator, seeded from one draw of
    ``rng`` and i, so the result depends on the seed alone."""
    n = int(np.prod(shape))
    x = np.empty(n, dtype=np.float32)
    base = int(rng.integers(0, 2**63 - 1))

    def fill(lo, hi):
        g = np.random.default_rng([base, lo // _CHUNK])
        g.standard_normal(size=hi - lo, dtype=np.float32, out=x[lo:hi])

    _chunked(n, fill)
    x = x.reshape(shape)
    return x if dtype == "f32" else f32_to_bf16_bits(x)


def e4m3_codes(rng: np.random.Generator, shape) -> np.ndarray:
    """Random fp8 e4m3 codes (uint8): random sign, exponent field 0..15 (every
    binade, subnormals and the top one up to 448 included), random mantissa;
    the two NaN codes (S.1111.111) are redrawn as the largest finite magnitude
    of the same sign, so a code is never NaN."""
    sign = rng.integers(0, 2, size=shape, dtype=np.uint8) << 7
    exp = rng.integers(0, 16, size=shape, dtype=np.uint8) << 3
    man = rng.integers(0, 8, size=shape, dtype=np.uint8)
    codes = (sign | exp | man).astype(np.uint8)
    nan = (codes & 0x7F) == 0x7F
    codes[nan] ^= 1  # 0x7F -> 0x7E (448), 0xFF -> 0xFE (-448)
    return codes


def e4m3_scales(rng: np.random.Generator, num_kv_heads: int) -> np.ndarray:
    """Per-kv-head dequantisation scales U(0.01, 0.1): with codes over the whole
    e4m3 range the stored values reach +-44.8, and an N(0,1) token appended at
    the smallest scale saturates only beyond |x| = 4.48."""
    return rng.uniform(0.01, 0.1, size=num_kv_heads).astype(np.float32)


def _cache_values(rng, shape, dtype: str) -> np.ndarray:
    """Stored cache contents: values for fp32/bf16 caches, codes for fp8."""
    return e4m3_codes(rng, shape) if dtype == "fp8" else _normal(rng, shape, dtype)


def _empty_cache(shape, dtype: str, poison: bool) -> np.ndarray:
    if dtype == "f32":
        return np.full(shape, np.nan if poison else 0.0, dtype=np.float32)
    if dtype == "fp8":
        return np.full(shape, E4M3_NAN if poison else 0, dtype=np.uint8)
    return np.full(shape, BF16_NAN if poison else 0, dtype=np.uint16)


def _fill_history(rng, k_cache, v_cache, table_row, n_tokens, bs, dtype, kv=None):
    """Write n_tokens random K/V rows at logical positions 0..n_tokens-1
    (``kv``: the rows, [n_tokens, Hkv, d] each, if already drawn)."""
    Hkv, d = k_cache.shape[1], k_cache.shape[3]
    if n_tokens <= 0:
        return
    if kv is None:
        kh = _cache_values(rng, (n_tokens, Hkv, d), dtype)
        vh = _cache_values(rng, (n_tokens, Hkv, d), dtype)
    else:
        kh, vh = kv
    nfull = n_tokens // bs
    if nfull:
        blocks = np.asarray(table_row[:nfull], dtype=np.int64)
        # [nfull*bs, Hkv, d] -> [nfull, bs, Hkv, d] -> [nfull, Hkv, bs, d]
        k_cache[blocks] = kh[: nfull * bs].reshape(nfull, bs, Hkv, d).transpose(0, 2, 1, 3)
        v_cache[blocks] = vh[: nfull * bs].reshape(nfull, bs, Hkv, d).transpose(0, 2, 1, 3)
    rem = n_tokens - nfull * bs
    if rem:
        p = int(table_row[nfull])
        k_cache[p, :, :rem, :] = kh[nfull * bs:].transpose(1, 0, 2)
        v_cache[p, :, :rem, :] = vh[nfull * bs:].transpose(1, 0, 2)


def make_paged(seq_lens, *, Hq: int, Hkv: int, d: int, bs: int, dtype: str, seed: int,
               pool_factor: float = 1.0, extra_blocks: int = 0, permute: bool = True,
               poison: bool = True, scale: float | None = None, name: str = "custom",
               append_last: bool = True, table_pad: int = 0) -> Workload:
    """Generic paged workload: each request owns ceil(L/bs) blocks taken in
    order from a (seeded, optionally permuted) pool; history tokens 0..L-2 are
    in the cache and token L-1 is the step's new token (``append_last``), or
    all L tokens are in the cache (``append_last=False``, no new tokens)."""
    rng = np.random.default_rng(seed)
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    B = int(seq_lens.shape[0])
    # fp8 caches: q and the appended tokens are bf16, the cache holds e4m3 codes
    qdt = "bf16" if dtype == "fp8" else dtype
    nblk = [-(-int(L) // bs) for L in seq_lens]
    need = int(sum(nblk))
    NB = max(int(math.ceil(need * pool_factor)) + int(extra_blocks), 1)
    pool = rng.permutation(NB) if permute else np.arange(NB)
    max_blocks = max(max(nblk) if nblk else 1, 1) + int(table_pad)
    tables = np.full((B, max_blocks), -1, dtype=np.int32)
    pos = 0
    for b in range(B):
        tables[b, : nblk[b]] = pool[pos: pos + nblk[b]]
        pos += nblk[b]
    q = _normal(rng, (B, Hq, d), qdt)
    k_cache = _empty_cache((NB, Hkv, bs, d), dtype, poison)
    v_cache = _empty_cache((NB, Hkv, bs, d), dtype, poison)
    hist = [int(L) - 1 if (append_last and L > 0) else int(L) for L in seq_lens]
    # every request's history rows in one draw (threaded), then laid out
    total = int(sum(hist))
    kh = _cache_values(rng, (total, Hkv, d), dtype)
    vh = _cache_values(rng, (total, Hkv, d), dtype)
    at = 0
    for b in range(B):
        n = hist[b]
        _fill_history(rng, k_cache, v_cache, tables[b], n, bs, dtype,
                      kv=(kh[at:at + n], vh[at:at + n]))
        at += n
    del kh, vh
    new_rows = [b for b in range(B) if append_last and seq_lens[b] > 0]
    T = len(new_rows)
    k_new = _normal(rng, (T, Hkv, d), qdt)
    v_new = _normal(rng, (T, Hkv, d), qdt)
    slots = np.zeros(T, dtype=np.int64)
    for i, b in enumerate(new_rows):
        t = int(seq_lens[b]) - 1
        slots[i] = int(tables[b, t // bs]) * bs + t % bs
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    ks = vs = None
    if dtype == "fp8":  # per-kv-head dequantisation scales
        ks = e4m3_scales(rng, Hkv)
        vs = e4m3_scales(rng, Hkv)
    return Workload(name=name, B=B, Hq=Hq, Hkv=Hkv, d=d, bs=bs, num_blocks=NB,
                    dtype=dtype, scale=float(scale), q=q, k_cache=k_cache,
                    v_cache=v_cache, block_tables=tables, seq_lens=seq_lens,
                    k_new=k_new, v_new=v_new, slot_mapping=slots,
                    info={"seed": seed, "blocks_used": need}, k_scale=ks, v_scale=vs)


def tiny_f32(poison: bool = True, seed: int = 1001) -> Workload:
    """batch 4, seq_lens [1,17,100,200], 4 q / 2 KV heads, d 64, block 16,
    pool of 64 blocks assigned by a seeded permutation, fp32, scale 1/8."""
    return make_paged([1, 17, 100, 200], Hq=4, Hkv=2, d=64, bs=16, dtype="f32",
                      seed=seed, extra_blocks=64 - 23, poison=poison,
                      scale=1.0 / 8.0, name="tiny_f32")


def gqa_4k(poison: bool = True, seed: int = 1002, batch: int = 16,
           seq_len: int = 4096) -> Workload:
    """batch 16 x 4096 tokens, 32 q / 8 KV heads, d 128, block 16, bf16; the
    4096 blocks are a random permutation of the pool split in order."""
    return make_paged([seq_len] * batch, Hq=32, Hkv=8, d=128, bs=16, dtype="bf16",
                      seed=seed, poison=poison, name="gqa_4k")


def mixed_lengths(seed: int = 1003, batch: int = 256, lo: int = 16, hi: int = 8192) -> np.ndarray:
    rng = np.random.default_rng(seed + 7919)
    u = rng.uniform(math.log(lo), math.log(hi), size=batch)
    return np.clip(np.floor(np.exp(u)), lo, hi).astype(np.int32)


def mixed(poison: bool = True, seed: int = 1003, batch: int = 256) -> Workload:
    """256 requests, log-uniform lengths in [16, 8192], 32 q / 8 KV heads,
    d 128, block 16, shuffled pool of 1.1x the blocks needed, bf16."""
    lens = mixed_lengths(seed, batch)
    return make_paged(lens, Hq=32, Hkv=8, d=128, bs=16, dtype="bf16", seed=seed,
                      pool_factor=1.1, poison=poison, name="mixed")


def prefix_shared(poison: bool = True, seed: int = 1004, batch: int = 64,
                  prefix_tokens: int = 2040, prefix_blocks: int = 128,
                  suffix_lo: int = 64, suffix_hi: int = 512, Hq: int = 32,
                  Hkv: int = 8, d: int = 128, bs: int = 16,
                  dtype: str = "bf16") -> Workload:
    """Requests whose block tables share one prefix held in ``prefix_blocks``
    physical blocks (the last partially filled).  Each request forks the last
    prefix block into a private block (copy_pairs), then appends its suffix
    (k_new / v_new / slot_mapping) starting inside the forked block."""
    assert (prefix_blocks - 1) * bs < prefix_tokens <= prefix_blocks * bs
    rng = np.random.default_rng(seed)
    suffix = rng.integers(suffix_lo, suffix_hi + 1, size=batch).astype(np.int64)
    fill_last = prefix_tokens - (prefix_blocks - 1) * bs  # tokens in the last prefix block
    # blocks per request: 1 fork + blocks after it
    extra = [(-(-(fill_last + int(s)) // bs)) - 1 for s in suffix]
    NB = prefix_blocks + batch + int(sum(extra))
    pool = rng.permutation(NB)
    shared = pool[:prefix_blocks]
    pos = prefix_blocks
    seq_lens = (prefix_tokens + suffix).astype(np.int32)
    max_blocks = int(max(-(-int(L) // bs) for L in seq_lens))
    tables = np.full((batch, max_blocks), -1, dtype=np.int32)
    pairs = np.zeros((batch, 2), dtype=np.int64)
    k_cache = _empty_cache((NB, Hkv, bs, d), dtype, poison)
    v_cache = _empty_cache((NB, Hkv, bs, d), dtype, poison)
    _fill_history(rng, k_cache, v_cache, shared, prefix_tokens, bs, dtype)
    slot_rows = []
    for b in range(batch):
        fork = int(pool[pos]); pos += 1
        own = [int(x) for x in pool[pos: pos + extra[b]]]; pos += extra[b]
        row = list(int(x) for x in shared[: prefix_blocks - 1]) + [fork] + own
        tables[b, : len(row)] = row
        pairs[b] = (int(shared[prefix_blocks - 1]), fork)
        for t in range(prefix_tokens, int(seq_lens[b])):
            slot_rows.append(row[t // bs] * bs + t % bs)
    T = len(slot_rows)
    k_new = _normal(rng, (T, Hkv, d), dtype)
    v_new = _normal(rng, (T, Hkv, d), dtype)
    q = _normal(rng, (batch, Hq, d), dtype)
    return Workload(name="prefix", B=batch, Hq=Hq, Hkv=Hkv, d=d, bs=bs, num_blocks=NB,
                    dtype=dtype, scale=1.0 / math.sqrt(d), q=q, k_cache=k_cache,
                    v_cache=v_cache, block_tables=tables, seq_lens=seq_lens,
                    k_new=k_new, v_new=v_new,
                    slot_mapping=np.asarray(slot_rows, dtype=np.int64),
                    copy_pairs=pairs,
                    info={"seed": seed, "prefix_tokens": prefix_tokens,
                          "prefix_blocks": [int(x) for x in shared],
                          "suffix": suffix.tolist()})


def prefix_groups(groups, singles: int = 0, *, seed: int = 1007, suffix_lo: int = 0,
                  suffix_hi: int = 300, Hq: int = 32, Hkv: int = 8, d: int = 128, bs: int = 16,
                  dtype: str = "bf16", poison: bool = True, short_members: int = 0,
                  interleave: bool = True) -> Workload:
    """Requests in groups that share the physical blocks of a prefix, plus
    ungrouped requests.  ``groups`` lists (members, prefix_tokens) with
    prefix_tokens a multiple of bs.  A member holds the group's shared blocks
    for its first prefix_tokens tokens, then its own blocks for a suffix of
    U{suffix_lo..suffix_hi} tokens; the first ``short_members`` members of each
    group instead stop inside the prefix (length U{1..prefix_tokens}).  The
    step appends each request's last token when it lies in a block of its own.
    ``interleave`` spreads members of different groups across the batch.
    info: prefix_of [B] int32 (-1 = none), prefix_lens [G] int32."""
    rng = np.random.default_rng(seed)
    reqs = []  # (group or -1, length)
    for g, (n, ptok) in enumerate(groups):
        assert ptok % bs == 0 and ptok >= 0
        for i in range(n):
            if i < short_members and ptok > 0:
                L = int(rng.integers(1, ptok + 1))
            else:
                L = ptok + int(rng.integers(suffix_lo, suffix_hi + 1))
            reqs.append((g, L))
    for _ in range(singles):
        reqs.append((-1, int(rng.integers(max(suffix_lo, 1), suffix_hi + 400))))
    if interleave:
        order = rng.permutation(len(reqs))
        reqs = [reqs[i] for i in order]
    B = len(reqs)
    shared_nb = [ptok // bs for _, ptok in groups]
    own_nb = []
    for g, L in reqs:
        nb = -(-L // bs)
        own_nb.append(max(nb - (shared_nb[g] if g >= 0 else 0), 0))
    NB = max(int(sum(shared_nb) + sum(own_nb)), 1)
    pool = rng.permutation(NB)
    pos = 0
    shared = []
    for nb in shared_nb:
        shared.append([int(x) for x in pool[pos: pos + nb]])
        pos += nb
    max_blocks = max(max(-(-L // bs) for _, L in reqs), 1)
    tables = np.full((B, max_blocks), -1, dtype=np.int32)
    qdt = "bf16" if dtype == "fp8" else dtype
    k_cache = _empty_cache((NB, Hkv, bs, d), dtype, poison)
    v_cache = _empty_cache((NB, Hkv, bs, d), dtype, poison)
    for g, ptok in enumerate(p for _, p in groups):
        _fill_history(rng, k_cache, v_cache, np.asarray(shared[g], np.int64), ptok, bs, dtype)
    slots = []
    new_rows = []
    for b, (g, L) in enumerate(reqs):
        nb = -(-L // bs)
        sh = shared[g] if g >= 0 else []
        own = [int(x) for x in pool[pos: pos + own_nb[b]]]
        pos += own_nb[b]
        row = (sh + own)[:nb]
        tables[b, : len(row)] = row
        first_own = len(sh) * bs  # first token in an own block
        last_in_own = L - 1 >= first_own
        hist_end = L - 1 if last_in_own else L
        # the request's own history tokens [first_own, hist_end)
        if hist_end > first_own:
            n_own = hist_end - first_own
            kh = _cache_values(rng, (n_own, Hkv, d), dtype)
            vh = _cache_values(rng, (n_own, Hkv, d), dtype)
            for i in range(n_own):
                t = first_own + i
                blk, off = row[t // bs], t % bs
                k_cache[blk, :, off, :] = kh[i]
                v_cache[blk, :, off, :] = vh[i]
        if last_in_own:
            t = L - 1
            slots.append(row[t // bs] * bs + t % bs)
            new_rows.append(b)
    T = len(slots)
    k_new = _normal(rng, (T, Hkv, d), qdt)
    v_new = _normal(rng, (T, Hkv, d), qdt)
    q = _normal(rng, (B, Hq, d), qdt)
    ks = vs = None
    if dtype == "fp8":
        ks = e4m3_scales(rng, Hkv)
        vs = e4m3_scales(rng, Hkv)
    return Workload(name="prefix_groups", B=B, Hq=Hq, Hkv=Hkv, d=d, bs=bs, num_blocks=NB,
                    dtype=dtype, scale=1.0 / math.sqrt(d), q=q, k_cache=k_cache,
                    v_cache=v_cache, block_tables=tables,
                    seq_lens=np.asarray([L for _, L in reqs], np.int32), k_new=k_new,
                    v_new=v_new, slot_mapping=np.asarray(slots, np.int64),
                    info={"seed": seed,
                          "prefix_of": np.asarray([g for g, _ in reqs], np.int32),
                          "prefix_lens": np.asarray([p for _, p in groups], np.int32)},
                    k_scale=ks, v_scale=vs)


def long_ctx(bs: int = 16, poison: bool = True, seed: int = 1005, batch: int = 2,
             seq_len: int = 131072) -> Workload:
    """batch 2 x 131072 tokens, 64 q / 8 KV heads, d 128, block size bs, bf16."""
    return make_paged([seq_len] * batch, Hq=64, Hkv=8, d=128, bs=bs, dtype="bf16",
                      seed=seed + bs, poison=poison, name=f"long_ctx_bs{bs}")


def gqa_4k_fp8(poison: bool = True, seed: int = 1006, batch: int = 16,
               seq_len: int = 4096) -> Workload:
    """The 4k-token decode workload with an fp8 (e4m3) cache: random codes with
    per-kv-head scales; q and appended tokens bf16."""
    return make_paged([seq_len] * batch, Hq=32, Hkv=8, d=128, bs=16, dtype="fp8",
                      seed=seed, poison=poison, name="gqa_4k_fp8")


WORKLOADS = {
    "tiny_f32": tiny_f32,
    "gqa_4k": gqa_4k,
    "mixed": mixed,
    "prefix": prefix_shared,
    "long_ctx": long_ctx,
    "gqa_4k_fp8": gqa_4k_fp8,
}
