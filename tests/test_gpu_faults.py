"""Device-detected faults and host validation that needs a device.

Bad indices are planted on the HOST in the inputs (a slot past the pool, a
block id past the pool, a sequence longer than its table, a copy pair out of
range).  The kernels must skip the bad item, raise a bit in the error word and
carry on -- no trap, no assert, no hang.  Nothing here faults the GPU."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workloads
from _helpers import DevWorkload, assert_decode_close, host_step, to_dev, to_host_f64

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkv():
    import paged_kv_cache_412_b200 as m
    m.get_device_error()  # start clean
    return m


def test_bad_slot_is_skipped_and_flagged(pkv):
    w = workloads.make_paged([10, 20, 30], Hq=4, Hkv=2, d=64, bs=16, dtype="bf16", seed=1)
    dw = DevWorkload(w)
    slots = dw.slot_mapping.clone()
    slots[1] = w.num_blocks * w.bs + 5
    before = dw.k_cache.clone()
    pkv.kv_cache_write(dw.k_new, dw.v_new, slots, dw.k_cache, dw.v_cache)
    assert pkv.get_device_error() & pkv.DEVERR["BAD_SLOT"]
    assert pkv.get_device_error() == 0  # read-and-clear
    # the two good tokens landed, nothing else changed
    kc_ref = w.k_cache.copy()
    vc_ref = w.v_cache.copy()
    good = np.array([0, 2])
    oracle.kv_cache_write(w.k_new[good], w.v_new[good], w.slot_mapping[good], kc_ref, vc_ref)
    got = dw.k_cache.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, kc_ref)


def test_bad_block_id_is_skipped_and_flagged(pkv):
    w = workloads.make_paged([100, 64, 50], Hq=8, Hkv=2, d=128, bs=16, dtype="bf16", seed=2,
                             append_last=False)
    bt = w.block_tables.copy()
    bt[1, 2] = w.num_blocks + 7  # request 1's third block is out of range
    dw = DevWorkload(w)
    out = pkv.paged_attention_decode(dw.q, dw.k_cache, dw.v_cache, to_dev(bt), dw.seq_lens,
                                     w.bs, w.scale)
    assert pkv.get_device_error() & pkv.DEVERR["BAD_BLOCK"]
    ref = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale)
    got = to_host_f64(out)
    for b in (0, 2):  # the other requests are untouched
        assert_decode_close(got[b], ref[b], "bf16", "bf16", what=f"req {b}")
    assert np.all(np.isfinite(got[1]))


def test_seq_len_past_table_is_clamped_and_flagged(pkv):
    w = workloads.make_paged([40, 16], Hq=4, Hkv=4, d=64, bs=16, dtype="f32", seed=3,
                             append_last=False)
    sl = w.seq_lens.copy()
    sl[1] = 10_000  # table holds 3 blocks (48 tokens) for this batch
    dw = DevWorkload(w)
    pkv.paged_attention_decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, to_dev(sl),
                               w.bs, w.scale)
    assert pkv.get_device_error() & pkv.DEVERR["BAD_SEQ_LEN"]


def test_bad_copy_pair_is_skipped_and_flagged(pkv):
    w = workloads.make_paged([40, 40], Hq=4, Hkv=2, d=64, bs=16, dtype="bf16", seed=4,
                             extra_blocks=4, append_last=False)
    pairs = np.array([[int(w.block_tables[0, 0]), w.num_blocks - 1], [0, w.num_blocks + 3]],
                     np.int64)
    dw = DevWorkload(w)
    pkv.copy_blocks(dw.k_cache, dw.v_cache, to_dev(pairs))
    assert pkv.get_device_error() & pkv.DEVERR["BAD_PAIR"]
    kc_ref, vc_ref = w.k_cache.copy(), w.v_cache.copy()
    oracle.copy_blocks(kc_ref, vc_ref, pairs[:1])
    got = dw.k_cache.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, kc_ref)


def test_workspace_too_small_is_rejected(pkv):
    w = workloads.make_paged([40], Hq=4, Hkv=2, d=64, bs=16, dtype="bf16", seed=5)
    dw = DevWorkload(w)
    tiny = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(pkv.PkvError) as ei:
        pkv.paged_attention_decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens,
                                   w.bs, w.scale, workspace=tiny)
    assert ei.value.status == 3


def test_clean_run_leaves_no_flag(pkv):
    w = workloads.make_paged([40, 7], Hq=4, Hkv=2, d=64, bs=16, dtype="bf16", seed=6)
    dw = DevWorkload(w)
    pkv.kv_cache_write(dw.k_new, dw.v_new, dw.slot_mapping, dw.k_cache, dw.v_cache)
    pkv.paged_attention_decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens,
                               w.bs, w.scale)
    assert pkv.get_device_error() == 0


@pytest.mark.parametrize("dtype,bs", [("bf16", 16), ("fp8", 16), ("bf16", 4), ("bf16", 2)])
def test_bad_block_tokens_do_not_take_part(pkv, dtype, bs):
    """A table entry outside the pool: that block's tokens are left out of the
    request's softmax (the others are unaffected) and PKV_DEVERR_BAD_BLOCK is
    raised.  Expected values: numpy brute force over the rows that remain."""
    from oracle import brute
    w = workloads.make_paged([100, 64, 50], Hq=8, Hkv=2, d=128, bs=bs, dtype=dtype, seed=3,
                             append_last=False)
    bt = w.block_tables.copy()
    bad_blk = 32 // bs  # request 1's block holding token 32 (tokens 32 .. 32 + bs - 1)
    bt[1, bad_blk] = w.num_blocks + 7
    dw = DevWorkload(w)
    out = pkv.paged_attention_decode(dw.q, dw.k_cache, dw.v_cache, to_dev(bt), dw.seq_lens, bs,
                                     w.scale, out_dtype=torch.float32, k_scale=dw.k_scale,
                                     v_scale=dw.v_scale)
    assert pkv.get_device_error() & pkv.DEVERR["BAD_BLOCK"]
    got = to_host_f64(out)
    G = w.Hq // w.Hkv

    def rows(cache, scale_arr, b, h, tokens):
        r = np.stack([cache[w.block_tables[b, t // bs], h, t % bs] for t in tokens])
        if dtype == "fp8":
            return workloads_e4m3(r) * float(scale_arr[h])
        return brute.bf16_bits_to_f64(r)

    q = brute.bf16_bits_to_f64(w.q)
    for b in range(3):
        L = int(w.seq_lens[b])
        keep = [t for t in range(L) if not (b == 1 and 32 <= t < 32 + bs)]
        for hq in range(w.Hq):
            h = hq // G
            ref = brute.attention_numpy(q[b, hq], rows(w.k_cache, w.k_scale, b, h, keep),
                                        rows(w.v_cache, w.v_scale, b, h, keep), w.scale)
            assert np.max(np.abs(got[b, hq] - ref)) <= 2e-3, (b, hq)


def workloads_e4m3(codes: np.ndarray) -> np.ndarray:
    """e4m3 codes -> float64 through torch's float8_e4m3fn (pinned against the
    oracle's code table in the oracle tests)."""
    t = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


# ---- bounded waits that run out (the fault is armed on the host) -------------
#
# The pages' own failure case is running out of blocks mid-generation
# ("PagedAttention: Optimizing KV Cache Utilization in Large Language Models",
# "Conclusion").  In the kernels the failure to guard against is a wait that
# never ends.  Every in-kernel wait is bounded; these tests arm a test-only
# fault for ONE decode call (pkv_internal_decode_fault, exported but not in the
# public header) that makes one wait run out after a few milliseconds: the
# call must raise PKV_DEVERR_TIMEOUT and return, the context must stay usable,
# and after pkv_decode_workspace_init the same decode must match the oracle.

FAULT_MERGE_FLAG, FAULT_SKIP_STAGE = 1, 2


def _arm(pkv, mode, arg=0, wait_ns=5_000_000):
    import ctypes
    f = pkv._get_lib().pkv_internal_decode_fault
    f.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_ulonglong]
    f.restype = ctypes.c_int
    assert f(mode, arg, wait_ns) == 0


@pytest.mark.parametrize("mode,arg", [(FAULT_MERGE_FLAG, 0), (FAULT_SKIP_STAGE, 1)],
                         ids=["merger-ready-flag", "stage-full-barrier"])
def test_wait_runs_out_then_workspace_recovers(pkv, mode, arg):
    # long requests: every (request, kv head) is split over several units, so
    # mergers exist, and CTA 0 streams more than two stages
    w = workloads.make_paged([4096, 3000, 1, 2500], Hq=32, Hkv=8, d=128, bs=16, dtype="bf16",
                             seed=61)
    dw = DevWorkload(w)
    pkv.kv_cache_write(dw.k_new, dw.v_new, dw.slot_mapping, dw.k_cache, dw.v_cache)
    L = int(w.seq_lens.max())
    ws = pkv.new_workspace(pkv.decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.d, w.bs, L, 0))
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    assert pkv.get_device_error() == 0
    _arm(pkv, mode, arg)
    pkv.paged_attention_decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.bs,
                               w.scale, out, max_seq_len=L, workspace=ws)
    flags = pkv.get_device_error()  # synchronises: the call has returned
    assert flags & pkv.DEVERR["TIMEOUT"], hex(flags)
    # the context is usable; a TIMEOUT leaves the workspace's counters and
    # flags in an unknown state, so re-initialise it, then decode again
    pkv.workspace_init(ws)
    pkv.paged_attention_decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.bs,
                               w.scale, out, max_seq_len=L, workspace=ws)
    assert pkv.get_device_error() == 0
    kc, vc = host_step(w)
    ref = oracle.decode(w.q, kc, vc, w.block_tables, w.seq_lens, w.scale)
    assert_decode_close(to_host_f64(out), ref, "bf16", "f32", what="decode after recovery")
    # the fault was consumed by the one call: the next call is clean too
    pkv.paged_attention_decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens, w.bs,
                               w.scale, out, max_seq_len=L, workspace=ws)
    assert pkv.get_device_error() == 0


def test_copy_contract_violation_is_flagged(pkv):
    """copy_blocks pairs must name distinct destinations, none of them also a
    source; a call that breaks it raises PKV_DEVERR_BAD_PAIR (its result is
    unspecified, so only the flag is checked), and a valid call does not."""
    w = workloads.make_paged([40, 40], Hq=4, Hkv=2, d=64, bs=16, dtype="bf16", seed=9,
                             extra_blocks=8, append_last=False)
    dw = DevWorkload(w)
    free = [b for b in range(w.num_blocks) if b not in set(w.block_tables[w.block_tables >= 0])]
    a, b = int(w.block_tables[0, 0]), int(w.block_tables[1, 0])
    for pairs in ([[a, free[0]], [b, free[0]]],      # destination repeated
                  [[a, free[0]], [free[0], free[1]]],  # a destination is also a source
                  [[a, a]]):                          # a block copied onto itself
        pkv.copy_blocks(dw.k_cache, dw.v_cache, to_dev(np.array(pairs, np.int64)))
        assert pkv.get_device_error() & pkv.DEVERR["BAD_PAIR"], pairs
    pkv.copy_blocks(dw.k_cache, dw.v_cache,
                    to_dev(np.array([[a, free[0]], [b, free[1]]], np.int64)))
    assert pkv.get_device_error() == 0
