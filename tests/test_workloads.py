"""The seeded input generators: shapes, structure and internal consistency
(no GPU).  The generators carry none of the method's arithmetic; these tests
check that the layouts they build are what the workloads describe."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workloads


def _check_consistent(w):
    assert w.q.shape == (w.B, w.Hq, w.d)
    assert w.k_cache.shape == (w.num_blocks, w.Hkv, w.bs, w.d) == w.v_cache.shape
    assert w.block_tables.dtype == np.int32 and w.seq_lens.dtype == np.int32
    used = []
    for b in range(w.B):
        n = -(-int(w.seq_lens[b]) // w.bs)
        row = w.block_tables[b, :n]
        assert np.all((row >= 0) & (row < w.num_blocks))
        assert np.all(w.block_tables[b, n:] == -1)
        used.append(row)
    for t, s in enumerate(w.slot_mapping):
        assert 0 <= s < w.num_blocks * w.bs


def test_tiny_f32_shapes():
    w = workloads.tiny_f32()
    assert w.num_blocks == 64 and w.B == 4 and list(w.seq_lens) == [1, 17, 100, 200]
    _check_consistent(w)
    assert w.k_new.shape == (4, 2, 64)
    # each new token goes to position L-1 of its request
    for b in range(4):
        t = int(w.seq_lens[b]) - 1
        assert w.slot_mapping[b] == w.block_tables[b, t // 16] * 16 + t % 16
        # that slot is still poisoned before the step
        p, o = divmod(int(w.slot_mapping[b]), 16)
        assert np.all(np.isnan(w.k_cache[p, :, o]))
    # blocks are all distinct (no sharing in this workload)
    flat = np.concatenate([w.block_tables[b, : -(-int(w.seq_lens[b]) // 16)] for b in range(4)])
    assert len(set(flat.tolist())) == len(flat) == 23


def test_tiny_f32_runs_through_the_oracle():
    w = workloads.tiny_f32()
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    assert oracle.kv_cache_write(w.k_new, w.v_new, w.slot_mapping, kc, vc) == 0
    out = oracle.decode(w.q, kc, vc, w.block_tables, w.seq_lens, w.scale)
    assert np.all(np.isfinite(out))
    # request 0 has one token: its output is the appended V row exactly
    for h in range(4):
        np.testing.assert_array_equal(out[0, h], w.v_new[0, h // 2].astype(np.float64))


def test_prefix_structure():
    w = workloads.prefix_shared(batch=6, suffix_lo=5, suffix_hi=40, Hq=4, Hkv=2, d=64)
    _check_consistent(w)
    shared = w.info["prefix_blocks"]
    for b in range(w.B):
        assert list(w.block_tables[b, :127]) == shared[:127]
        assert w.block_tables[b, 127] != shared[127]
        assert tuple(w.copy_pairs[b]) == (shared[127], w.block_tables[b, 127])
    assert w.slot_mapping.shape[0] == sum(w.info["suffix"])
    assert len(set(w.slot_mapping.tolist())) == len(w.slot_mapping)


def test_mixed_lengths_distribution():
    lens = workloads.mixed_lengths(1003, 256)
    assert lens.min() >= 16 and lens.max() <= 8192
    assert 600 < lens.mean() < 2200  # log-uniform on [16, 8192]: mean ~1311


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.00390625, 1.005859375, 1.0078125, -2.5], np.float32)
    bits = workloads.f32_to_bf16_bits(x)
    back = workloads.bf16_bits_to_f32(bits)
    np.testing.assert_array_equal(back, [1.0, 1.0, 1.0078125, 1.0078125, -2.5])


@pytest.mark.parametrize("permute", [True, False])
def test_make_paged_tail_and_pool(permute):
    w = workloads.make_paged([0, 5, 33], Hq=4, Hkv=4, d=64, bs=8, dtype="bf16", seed=3,
                             pool_factor=1.5, permute=permute, table_pad=2)
    _check_consistent(w)
    assert w.block_tables.shape[1] == 5 + 2
    assert w.k_new.shape[0] == 2  # the empty request appends nothing


def test_prefix_groups_share_blocks_and_fill_every_token():
    """Members of a group name the same physical blocks for the prefix; after
    the step (append of each request's last token) every token below a
    request's length is a value, never the poison; appended slots lie in
    blocks of the request's own."""
    w = workloads.prefix_groups([(5, 64), (3, 128), (4, 0)], singles=3, bs=16, Hq=8, Hkv=2,
                                d=64, short_members=1, seed=3)
    po, pl = w.info["prefix_of"], w.info["prefix_lens"]
    for g in range(len(pl)):
        mem = np.where(po == g)[0]
        nb = pl[g] // w.bs
        longest = max(mem, key=lambda b: w.seq_lens[b])
        for b in mem:
            n = min(nb, -(-int(w.seq_lens[b]) // w.bs))
            assert np.array_equal(w.block_tables[b, :n], w.block_tables[longest, :n])
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    for i, s in enumerate(w.slot_mapping):
        kc[s // w.bs, :, s % w.bs] = w.k_new[i]
        vc[s // w.bs, :, s % w.bs] = w.v_new[i]
    shared = {int(x) for g in range(len(pl)) for x in
              w.block_tables[np.where(po == g)[0][0], : pl[g] // w.bs]}
    for s in w.slot_mapping:
        assert int(s) // w.bs not in shared
    for b in range(w.B):
        for t in range(int(w.seq_lens[b])):
            blk = w.block_tables[b, t // w.bs]
            assert blk >= 0
            assert not np.any(kc[blk, :, t % w.bs] == workloads.BF16_NAN)
            assert not np.any(vc[blk, :, t % w.bs] == workloads.BF16_NAN)


def test_e4m3_codes_cover_every_binade_and_never_nan():
    """The fp8 history draws every exponent field 0..15 (subnormals up to the
    binade of 448) with both signs, and never a NaN code (S.1111.111)."""
    codes = workloads.e4m3_codes(np.random.default_rng(5), (64, 1024))
    assert not np.any((codes & 0x7F) == 0x7F)
    assert set(np.unique((codes >> 3) & 0xF).tolist()) == set(range(16))
    assert set(np.unique(codes >> 7).tolist()) == {0, 1}
    assert np.any(codes == 0x7E) and np.any(codes == 0xFE)  # +-448
