"""Prefix-aware decode (GPU): requests that share a prefix's physical blocks
read them once per group ("KV Cache Management", "The Bonus: Zero-Copy
Sharing").  The result must be the plain attention over each request's full
block table, so every case compares pkv_paged_attention_decode_prefix with the
oracle's plain definition on the same tables (bf16 tolerance as for decode)."""
from __future__ import annotations

import math

import numpy as np
import pytest

import oracle
import workloads
from _helpers import DevWorkload, assert_decode_close, host_step, to_dev, to_host_f64

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _run(w, prefix_of, prefix_lens, out_dtype, max_members=None, max_prefix_len=None,
         step=True):
    import paged_kv_cache_412_b200 as pkv
    dw = DevWorkload(w)
    if step:
        if w.copy_pairs.shape[0]:
            pkv.copy_blocks(dw.k_cache, dw.v_cache, dw.copy_pairs)
        if w.slot_mapping.shape[0]:
            pkv.kv_cache_write(dw.k_new, dw.v_new, dw.slot_mapping, dw.k_cache, dw.v_cache)
    out = pkv.paged_attention_decode_prefix(
        dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens,
        to_dev(np.asarray(prefix_of, np.int32)), to_dev(np.asarray(prefix_lens, np.int32)),
        w.bs, w.scale, out_dtype=out_dtype, max_prefix_members=max_members,
        max_prefix_len=max_prefix_len)
    torch.cuda.synchronize()
    return to_host_f64(out), pkv.get_device_error()


def _oracle(w):
    kc, vc = host_step(w)
    return oracle.decode(w.q, kc, vc, w.block_tables, w.seq_lens, w.scale)


@pytest.mark.parametrize("out_dtype", ["bf16", "f32"])
def test_shared_prefix_workload(out_dtype):
    """64 requests forked from a 2040-token prompt: 127 shared full blocks
    (2032 tokens) read once per group; the forked block 127 and the suffixes
    in each request's own pass."""
    w = workloads.prefix_shared(poison=True)
    ref = _oracle(w)
    tdt = torch.bfloat16 if out_dtype == "bf16" else torch.float32
    got, err = _run(w, np.zeros(w.B, np.int32), [2032], tdt, max_members=64, max_prefix_len=2040)
    assert err == 0
    assert_decode_close(got, ref, "bf16", out_dtype, what="prefix workload")


CASES = [
    # (bs, Hq, Hkv, d, groups, singles, short)
    (16, 32, 8, 128, [(9, 256), (1, 64), (5, 1024), (3, 0)], 3, 2),
    (8, 32, 8, 128, [(7, 200), (4, 64)], 2, 1),
    (32, 16, 8, 64, [(6, 512), (2, 96)], 2, 1),
    (128, 32, 8, 128, [(5, 384), (3, 128)], 1, 1),
    (16, 32, 2, 128, [(6, 320), (2, 64)], 1, 1),   # 16 query heads per kv head
    (16, 24, 8, 64, [(23, 192), (5, 48)], 2, 2),   # 3 query heads per kv head
    (16, 64, 8, 128, [(40, 448), (3, 32)], 1, 2),  # 320 rows: three 128-row tiles, the last partial
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"bs{c[0]}-G{c[1] // c[2]}-d{c[3]}")
def test_prefix_groups(case):
    bs, Hq, Hkv, d, groups, singles, short = case
    groups = [(n, (p // bs) * bs) for n, p in groups]
    w = workloads.prefix_groups(groups, singles, bs=bs, Hq=Hq, Hkv=Hkv, d=d,
                                short_members=short, seed=1100 + bs + d + Hq)
    ref = _oracle(w)
    got, err = _run(w, w.info["prefix_of"], w.info["prefix_lens"], torch.bfloat16)
    assert err == 0
    assert_decode_close(got, ref, "bf16", "bf16", what=f"groups {case}")
    got32, err = _run(w, w.info["prefix_of"], w.info["prefix_lens"], torch.float32)
    assert err == 0
    assert_decode_close(got32, ref, "bf16", "f32", what=f"groups {case} f32 out")


def test_member_whose_whole_length_is_the_prefix():
    """A member of exactly prefix_len tokens has no token of its own pass: its
    output is the merge of the shared pass's results alone."""
    w = workloads.prefix_groups([(4, 256)], 0, bs=16, Hq=8, Hkv=2, d=128, suffix_lo=0,
                                suffix_hi=0, seed=1201)
    assert np.all(w.seq_lens == 256)
    ref = _oracle(w)
    got, err = _run(w, w.info["prefix_of"], w.info["prefix_lens"], torch.float32)
    assert err == 0
    assert_decode_close(got, ref, "bf16", "f32", what="whole length in the prefix")


def test_long_member_suffix_splits_its_own_pass():
    """One member with a long suffix: its own pass spans several split units,
    so the prefix results are folded in by the unit that merges the group."""
    w = workloads.prefix_groups([(3, 512)], 0, bs=16, Hq=32, Hkv=8, d=128, suffix_lo=20000,
                                suffix_hi=30000, seed=1202)
    ref = _oracle(w)
    got, err = _run(w, w.info["prefix_of"], w.info["prefix_lens"], torch.float32)
    assert err == 0
    assert_decode_close(got, ref, "bf16", "f32", what="long suffix")


def test_prefix_length_not_whole_blocks_is_rounded_and_flagged():
    """A prefix length off a block boundary is rounded down (the shared pass
    covers fewer tokens, each request's own pass the rest), the result stays
    the plain attention, and the device flags PKV_DEVERR_PREFIX."""
    import paged_kv_cache_412_b200 as pkv
    w = workloads.prefix_groups([(5, 256)], 1, bs=16, Hq=8, Hkv=2, d=128, seed=1203)
    ref = _oracle(w)
    got, err = _run(w, w.info["prefix_of"], [256 + 5], torch.float32)
    assert err == pkv.DEVERR["PREFIX"]
    assert_decode_close(got, ref, "bf16", "f32", what="rounded prefix")


def test_group_id_out_of_range_is_flagged_and_decoded_plainly():
    import paged_kv_cache_412_b200 as pkv
    w = workloads.prefix_groups([(4, 128)], 2, bs=16, Hq=8, Hkv=2, d=128, seed=1204)
    ref = _oracle(w)
    po = w.info["prefix_of"].copy()
    po[po == 0] = 7  # no such group: those requests run as ungrouped
    got, err = _run(w, po, w.info["prefix_lens"], torch.float32)
    assert err == pkv.DEVERR["PREFIX"]
    assert_decode_close(got, ref, "bf16", "f32", what="bad group id")


def test_too_many_members_is_flagged():
    import paged_kv_cache_412_b200 as pkv
    w = workloads.prefix_groups([(40, 128)], 0, bs=16, Hq=8, Hkv=2, d=128, seed=1205)
    _, err = _run(w, w.info["prefix_of"], w.info["prefix_lens"], torch.float32, max_members=8)
    assert err & pkv.DEVERR["PREFIX"]


def test_unsupported_configurations_are_refused():
    import paged_kv_cache_412_b200 as pkv
    w = workloads.make_paged([40, 50], Hq=4, Hkv=2, d=64, bs=16, dtype="f32", seed=5)
    dw = DevWorkload(w)
    with pytest.raises(pkv.PkvError) as ei:
        pkv.paged_attention_decode_prefix(dw.q, dw.k_cache, dw.v_cache, dw.block_tables,
                                          dw.seq_lens, to_dev(np.zeros(2, np.int32)),
                                          to_dev(np.array([32], np.int32)))
    assert ei.value.status == 2
