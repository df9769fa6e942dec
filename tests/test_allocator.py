"""Host block allocator (C++ in libpkv.so): on-demand blocks, block tables,
reference-counted sharing and copy-on-write; waste accounting against the
figures the pages print.  No GPU."""
from __future__ import annotations

import numpy as np
import pytest

import paged_kv_cache_412_b200 as pkv
import workloads
from oracle import byte_model


class RefAllocator:
    """Plain-Python model of the same rules, written from the description:
    LIFO free list starting with block 0; a block per block_size tokens, taken
    when the previous one is full; fork shares every block; an append into a
    shared, partially filled last block first moves the sequence to a fresh
    copy of it."""

    def __init__(self, nb, bs):
        self.bs = bs
        self.free = list(range(nb - 1, -1, -1))
        self.ref = [0] * nb
        self.seqs = {}

    def add(self, s):
        self.seqs[s] = ([], 0)

    def fork(self, p, c):
        blocks, n = self.seqs[p]
        for b in blocks:
            self.ref[b] += 1
        self.seqs[c] = (list(blocks), n)

    def _take(self):
        b = self.free.pop()
        self.ref[b] = 1
        return b

    def _drop(self, b):
        self.ref[b] -= 1
        if self.ref[b] == 0:
            self.free.append(b)

    def append(self, s, k):
        blocks, n = self.seqs[s]
        part = n % self.bs
        cow = part != 0 and self.ref[blocks[-1]] > 1
        room = self.bs - part if part else 0
        need = -(-(k - room) // self.bs) if k > room else 0
        if len(self.free) < need + (1 if cow else 0):
            return None
        pair = None
        if cow:
            src, dst = blocks[-1], self._take()
            self._drop(src)
            blocks[-1] = dst
            pair = (src, dst)
        slots = []
        for i in range(k):
            t = n + i
            if t % self.bs == 0:
                blocks.append(self._take())
            slots.append(blocks[t // self.bs] * self.bs + t % self.bs)
        self.seqs[s] = (blocks, n + k)
        return slots, pair

    def free_seq(self, s):
        for b in self.seqs.pop(s)[0]:
            self._drop(b)


def test_appends_follow_the_block_table():
    a = pkv.BlockAllocator(32, 16)
    a.add_seq(7)
    slots, cow = a.append(7, 40)
    assert cow is None
    table, n = a.block_table(7)
    assert n == 40 and list(table) == [0, 1, 2]
    t = np.arange(40)
    assert np.array_equal(slots, table[t // 16] * 16 + t % 16)
    more, _ = a.append(7, 1)
    assert more[0] == table[2] * 16 + 8
    st = a.stats()
    assert st["used_blocks"] == 3 and st["free_blocks"] == 29 and st["unused_slots"] == 7


def test_fork_and_copy_on_write():
    bs = 16
    a = pkv.BlockAllocator(400, bs)
    a.add_seq(0)
    a.append(0, 2040)  # the shared prefix: 127 full blocks + 8 tokens in block 127
    prefix, _ = a.block_table(0)
    assert len(prefix) == 128
    for c in range(1, 4):
        a.fork(0, c)
    assert a.refcount(int(prefix[127])) == 4 and a.stats()["shared_blocks"] == 128
    slots, cow = a.append(1, 5)
    assert cow is not None and cow[0] == prefix[127]
    table1, n1 = a.block_table(1)
    assert n1 == 2045 and list(table1[:127]) == list(prefix[:127]) and table1[127] == cow[1]
    assert slots[0] == cow[1] * bs + 8  # continues at offset 8 of the private copy
    assert a.refcount(int(prefix[127])) == 3
    # the parent itself must also copy before writing while the block is shared
    _, cow0 = a.append(0, 1)
    assert cow0 is not None and cow0[0] == prefix[127]
    # a sequence whose last block is full appends without a copy
    a.fork(1, 9)
    a.append(9, 11)  # fills its (shared-with-1) block 127 ... after a copy
    _, cow9 = a.append(9, 3)
    assert cow9 is None


def test_out_of_blocks_changes_nothing():
    a = pkv.BlockAllocator(4, 16)
    a.add_seq(1)
    a.append(1, 50)  # 4 blocks
    before = a.stats()
    with pytest.raises(pkv.PkvError) as ei:
        a.append(1, 20)
    assert ei.value.status == 6
    assert a.stats() == before
    a.free_seq(1)
    assert a.stats()["free_blocks"] == 4


@pytest.mark.parametrize("seed", range(6))
def test_matches_reference_model_under_random_operations(seed):
    rng = np.random.default_rng(seed)
    nb, bs = 96, [1, 4, 16][seed % 3]
    a = pkv.BlockAllocator(nb, bs)
    ref = RefAllocator(nb, bs)
    live, next_id = [], 0
    for _ in range(400):
        op = rng.integers(0, 10)
        if op < 2 or not live:
            a.add_seq(next_id)
            ref.add(next_id)
            live.append(next_id)
            next_id += 1
        elif op < 3:
            p = int(rng.choice(live))
            a.fork(p, next_id)
            ref.fork(p, next_id)
            live.append(next_id)
            next_id += 1
        elif op < 4 and len(live) > 1:
            s = int(rng.choice(live))
            a.free_seq(s)
            ref.free_seq(s)
            live.remove(s)
        else:
            s = int(rng.choice(live))
            k = int(rng.integers(1, 3 * bs + 2))
            want = ref.append(s, k)
            if want is None:
                with pytest.raises(pkv.PkvError):
                    a.append(s, k)
            else:
                slots, cow = a.append(s, k)
                assert list(slots) == want[0] and cow == want[1]
        for s in live:
            table, n = a.block_table(s)
            assert list(table) == ref.seqs[s][0] and n == ref.seqs[s][1]
        assert a.stats()["free_blocks"] == len(ref.free)


def test_waste_figures_from_the_pages():
    # the 200-token request of the page's example: 3896 slots idle in a 4096
    # reservation, 8 (at most block_size - 1 = 15) with 16-slot blocks
    r = pkv.waste_compare([200], 4096, 16, 1 << 20)
    assert r["contiguous_reserved"] - r["used_slots"] == byte_model.unused_slots_contiguous(200, 4096) == 3896
    assert r["paged_reserved"] - r["used_slots"] == byte_model.unused_slots_paged(200, 16) == 8
    a = pkv.BlockAllocator(64, 16)
    a.add_seq(0)
    a.append(0, 200)
    assert a.stats()["unused_slots"] == 8


def test_waste_on_mixed_lengths_against_the_pages_claims():
    """The pages: contiguous reservation wastes 60-80% of KV memory, paging
    under ~4%.  With log-uniform lengths in [16, 8192] reserved at 8192, the
    contiguous waste lands at or above that range and the paged waste well
    under 4%; paging admits several times more requests into the same pool."""
    lens = workloads.mixed_lengths(1003, 256)
    r = pkv.waste_compare(lens, 8192, 16, 8192 * 64)
    contiguous = 1 - r["used_slots"] / r["contiguous_reserved"]
    paged = 1 - r["used_slots"] / r["paged_reserved"]
    assert contiguous > 0.6
    assert paged < 0.04
    assert r["contiguous_admitted"] == 64
    assert r["paged_admitted"] >= 2 * r["contiguous_admitted"]
