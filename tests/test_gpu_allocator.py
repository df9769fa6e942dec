"""The host block allocator driving the GPU path (GPU).

A shared prefix is written once, requests fork it, the allocator hands out the
copy-on-write pairs and the slots of each request's suffix, and the device runs
pkv_copy_blocks -> pkv_kv_cache_write -> pkv_paged_attention_decode on the
block tables it produced.  The same operations are replayed on the CPU oracle;
caches must agree bit for bit and decode within the bf16 tolerance."""
from __future__ import annotations

import math

import numpy as np
import pytest

import oracle
import workloads
from _helpers import assert_decode_close, to_dev, to_host_bits, to_host_f64

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def test_allocator_drives_fork_append_decode():
    import paged_kv_cache_412_b200 as pkv
    rng = np.random.default_rng(123)
    bs, Hq, Hkv, d, NB = 16, 8, 2, 128, 256
    a = pkv.BlockAllocator(NB, bs)
    kc = np.full((NB, Hkv, bs, d), workloads.BF16_NAN, np.uint16)
    vc = kc.copy()
    dk, dv = to_dev(kc), to_dev(vc)

    def write(slots, n):
        k = workloads.f32_to_bf16_bits(rng.standard_normal((n, Hkv, d), dtype=np.float32))
        v = workloads.f32_to_bf16_bits(rng.standard_normal((n, Hkv, d), dtype=np.float32))
        assert oracle.kv_cache_write(k, v, slots, kc, vc) == 0
        pkv.kv_cache_write(to_dev(k), to_dev(v), to_dev(slots.astype(np.int64)), dk, dv)

    a.add_seq(0)
    slots, _ = a.append(0, 1000)  # shared prefix, last block partially filled
    write(slots, 1000)
    children = list(range(1, 7))
    for c in children:
        a.fork(0, c)
    pairs, new_slots, counts = [], [], []
    for c in children:
        n = int(rng.integers(1, 90))
        s, cow = a.append(c, n)
        if cow is not None:
            pairs.append(cow)
        new_slots.append(s)
        counts.append(n)
    pairs = np.asarray(pairs, np.int64).reshape(-1, 2)
    assert len(pairs) == len(children)  # every child wrote into the shared tail block
    assert oracle.copy_blocks(kc, vc, pairs) == 0
    pkv.copy_blocks(dk, dv, to_dev(pairs))
    write(np.concatenate(new_slots), int(sum(counts)))
    torch.cuda.synchronize()
    assert np.array_equal(to_host_bits(dk), kc) and np.array_equal(to_host_bits(dv), vc)

    tables = [a.block_table(c) for c in children]
    maxb = max(len(t) for t, _ in tables)
    bt = np.full((len(children), maxb), -1, np.int32)
    for i, (t, _) in enumerate(tables):
        bt[i, : len(t)] = t
    sl = np.array([n for _, n in tables], np.int32)
    q = workloads.f32_to_bf16_bits(rng.standard_normal((len(children), Hq, d), dtype=np.float32))
    out = pkv.paged_attention_decode(to_dev(q), dk, dv, to_dev(bt), to_dev(sl), bs,
                                     1 / math.sqrt(d), out_dtype=torch.float32)
    ref = oracle.decode(q, kc, vc, bt, sl, 1 / math.sqrt(d))
    assert_decode_close(to_host_f64(out), ref, "bf16", "f32", what="allocator-driven step")
    assert pkv.get_device_error() == 0
