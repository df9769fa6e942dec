"""Pins for the CPU oracle (no GPU).

The oracle is trusted only because these tests tie it to things fixed outside
itself: a numpy and a pure-Python brute force on contiguous data, the
invariances the pages state for paging (any physical placement, any block
size, shared prefix blocks), closed forms, the figures the pages print, and a
mutation check that plants plausible mistakes in the oracle and requires the
pins to catch each one.
"""
from __future__ import annotations

import math
import os
import tempfile

import numpy as np
import pytest

import oracle
from oracle import brute, byte_model

RNG = np.random.default_rng(12345)


# ---------------------------------------------------------------------------
# helpers: place contiguous per-request K/V into a paged cache (test-side code,
# written independently of workloads.py and of the oracle's gather)
# ---------------------------------------------------------------------------

def paged_from_contiguous(Kc, Vc, bs, NB=None, perm=None, dtype=np.float32, fill=np.nan):
    """Kc/Vc: list over requests of arrays [L_b, Hkv, d].  Returns caches
    [NB, Hkv, bs, d], block table [B, maxblk] (-1 tail), seq_lens."""
    B = len(Kc)
    Hkv, d = Kc[0].shape[1], Kc[0].shape[2]
    lens = [k.shape[0] for k in Kc]
    nblk = [-(-L // bs) for L in lens]
    need = sum(nblk)
    NB = NB or max(need, 1)
    perm = np.arange(NB) if perm is None else np.asarray(perm)
    kc = np.full((NB, Hkv, bs, d), fill, dtype=dtype)
    vc = np.full((NB, Hkv, bs, d), fill, dtype=dtype)
    maxb = max(max(nblk), 1)
    tables = np.full((B, maxb), -1, dtype=np.int32)
    nxt = 0
    for b in range(B):
        for j in range(nblk[b]):
            p = int(perm[nxt]); nxt += 1
            tables[b, j] = p
            for o in range(bs):
                t = j * bs + o
                if t < lens[b]:
                    for g in range(Hkv):
                        kc[p, g, o, :] = Kc[b][t, g, :]
                        vc[p, g, o, :] = Vc[b][t, g, :]
    return kc, vc, tables, np.asarray(lens, dtype=np.int32)


def rand_problem(lens, Hq, Hkv, d, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((len(lens), Hq, d)).astype(np.float32)
    Kc = [rng.standard_normal((L, Hkv, d)).astype(np.float32) for L in lens]
    Vc = [rng.standard_normal((L, Hkv, d)).astype(np.float32) for L in lens]
    return q, Kc, Vc


def brute_all(q, Kc, Vc, scale):
    """Textbook attention per (b, h); q head h reads kv head h // (Hq // Hkv)."""
    B, Hq, d = q.shape
    Hkv = Kc[0].shape[1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, d))
    for b in range(B):
        for h in range(Hq):
            g = h // G
            out[b, h] = brute.attention_numpy(q[b, h], Kc[b][:, g, :], Vc[b][:, g, :], scale)
    return out


# ---------------------------------------------------------------------------
# brute force
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("lens,Hq,Hkv,d,bs", [
    ([1, 2, 5, 17], 4, 2, 8, 4),
    ([33, 16, 1, 40], 6, 3, 16, 8),
    ([100, 7], 8, 1, 64, 16),
    ([64], 2, 2, 128, 16),
])
def test_oracle_matches_numpy_brute_force(lens, Hq, Hkv, d, bs):
    q, Kc, Vc = rand_problem(lens, Hq, Hkv, d, seed=sum(lens) + d)
    NB = sum(-(-L // bs) for L in lens) + 5
    perm = np.random.default_rng(7).permutation(NB)
    kc, vc, bt, sl = paged_from_contiguous(Kc, Vc, bs, NB=NB, perm=perm)
    scale = 1.0 / math.sqrt(d)
    got = oracle.decode(q, kc, vc, bt, sl, scale)
    ref = brute_all(q, Kc, Vc, scale)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_oracle_matches_python_loops_tiny():
    lens = [3, 1, 2]
    q, Kc, Vc = rand_problem(lens, 2, 1, 4, seed=99)
    kc, vc, bt, sl = paged_from_contiguous(Kc, Vc, bs=2, NB=6, perm=[5, 0, 3, 2, 4, 1])
    got = oracle.decode(q, kc, vc, bt, sl, 0.7)
    for b, L in enumerate(lens):
        for h in range(2):
            ref = brute.attention_loops(q[b, h].tolist(), Kc[b][:, 0, :].tolist(),
                                        Vc[b][:, 0, :].tolist(), 0.7)
            np.testing.assert_allclose(got[b, h], ref, rtol=0, atol=1e-13)


def test_hand_indexed_gather():
    """Every cache row carries its own address; with q = 0 the output is the
    plain mean of exactly the rows the block table names."""
    NB, Hkv, bs, d = 5, 2, 4, 4
    kc = np.zeros((NB, Hkv, bs, d), np.float32)
    vc = np.zeros((NB, Hkv, bs, d), np.float32)
    for p in range(NB):
        for g in range(Hkv):
            for o in range(bs):
                vc[p, g, o, :] = [p, g, o, 1000 * p + 100 * g + o]
    bt = np.array([[3, 0, -1], [4, -1, -1]], np.int32)
    sl = np.array([6, 1], np.int32)  # req0: block 3 (4 slots) + block 0 (2 slots)
    q = np.zeros((2, 4, d), np.float32)  # Hq = 4, G = 2
    out = oracle.decode(q, kc, vc, bt, sl, 1.0)
    for h in range(4):
        g = h // 2
        rows0 = [vc[3, g, o] for o in range(4)] + [vc[0, g, o] for o in range(2)]
        np.testing.assert_allclose(out[0, h], np.mean(rows0, axis=0), atol=1e-12)
        np.testing.assert_array_equal(out[1, h], vc[4, g, 0].astype(np.float64))


# ---------------------------------------------------------------------------
# invariances stated by the pages
# ---------------------------------------------------------------------------

def test_permutation_invariance():
    """The block table maps logical to physical blocks like a page table: any
    physical placement gives the same attention."""
    lens = [50, 3, 31, 64]
    q, Kc, Vc = rand_problem(lens, 4, 2, 16, seed=3)
    NB = 40
    ref = None
    for s in range(4):
        perm = np.random.default_rng(s).permutation(NB)
        kc, vc, bt, sl = paged_from_contiguous(Kc, Vc, 8, NB=NB, perm=perm)
        out = oracle.decode(q, kc, vc, bt, sl, 0.25)
        if ref is None:
            ref = out
        np.testing.assert_array_equal(out, ref)


@pytest.mark.parametrize("bs", [1, 8, 16, 32, 128])
def test_block_size_invariance(bs):
    lens = [1, 17, 100]
    q, Kc, Vc = rand_problem(lens, 4, 2, 32, seed=5)
    kc, vc, bt, sl = paged_from_contiguous(Kc, Vc, bs)
    out = oracle.decode(q, kc, vc, bt, sl, 0.2)
    kc1, vc1, bt1, sl1 = paged_from_contiguous(Kc, Vc, 1)
    ref = oracle.decode(q, kc1, vc1, bt1, sl1, 0.2)
    np.testing.assert_array_equal(out, ref)


def test_shared_prefix_equals_copied_prefix():
    """Block tables pointing at one physical copy of a shared prefix give the
    same result as every request holding its own copy."""
    rng = np.random.default_rng(11)
    bs, Hkv, Hq, d = 8, 2, 4, 16
    P = 3 * bs  # prefix fills 3 blocks
    pk = rng.standard_normal((P, Hkv, d)).astype(np.float32)
    pv = rng.standard_normal((P, Hkv, d)).astype(np.float32)
    suff = [5, 12, 1]
    Kc = [np.concatenate([pk, rng.standard_normal((s, Hkv, d)).astype(np.float32)]) for s in suff]
    Vc = [np.concatenate([pv, rng.standard_normal((s, Hkv, d)).astype(np.float32)]) for s in suff]
    q = rng.standard_normal((3, Hq, d)).astype(np.float32)
    # copied: every request owns its blocks
    kc, vc, bt, sl = paged_from_contiguous(Kc, Vc, bs)
    ref = oracle.decode(q, kc, vc, bt, sl, 0.3)
    # shared: point every request's first 3 table entries at request 0's blocks
    bt2 = bt.copy()
    bt2[1:, :3] = bt[0, :3]
    kc2, vc2 = kc.copy(), vc.copy()
    for b in (1, 2):
        kc2[bt[b, :3]] = np.nan  # the private prefix copies are now unused
        vc2[bt[b, :3]] = np.nan
    out = oracle.decode(q, kc2, vc2, bt2, sl, 0.3)
    np.testing.assert_array_equal(out, ref)


def test_partitioned_restatement_equals_plain():
    lens = [1, 9, 77, 130]
    q, Kc, Vc = rand_problem(lens, 4, 2, 16, seed=21)
    kc, vc, bt, sl = paged_from_contiguous(Kc, Vc, 8, NB=60,
                                           perm=np.random.default_rng(2).permutation(60))
    ref = oracle.decode(q, kc, vc, bt, sl, 0.25)
    for P in (1, 7, 8, 16, 100, 1000):
        got = oracle.decode_partitioned(q, kc, vc, bt, sl, 0.25, P)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------
# closed forms and special cases
# ---------------------------------------------------------------------------

def test_length_one_returns_v_row_exactly():
    q, Kc, Vc = rand_problem([1, 1], 4, 2, 32, seed=8)
    kc, vc, bt, sl = paged_from_contiguous(Kc, Vc, 16)
    out = oracle.decode(q, kc, vc, bt, sl, 0.5)
    for b in range(2):
        for h in range(4):
            np.testing.assert_array_equal(out[b, h], Vc[b][0, h // 2].astype(np.float64))


def test_weights_sum_to_one_and_nonnegative():
    q, Kc, Vc = rand_problem([37, 200], 4, 2, 16, seed=13)
    q *= 4.0  # peaky softmax
    kc, vc, bt, sl = paged_from_contiguous(Kc, Vc, 16)
    for b in range(2):
        for h in range(4):
            w = oracle.decode_weights(q, kc, vc, bt, sl, 0.5, b, h)
            assert w.shape == (int(sl[b]),)
            assert np.all(w >= 0)
            assert abs(math.fsum(w) - 1.0) <= 1e-12


def test_zero_query_and_zero_scale_give_mean_of_v():
    q, Kc, Vc = rand_problem([13, 40], 2, 2, 8, seed=4)
    kc, vc, bt, sl = paged_from_contiguous(Kc, Vc, 8)
    for qq, sc in ((np.zeros_like(q), 0.5), (q, 0.0)):
        out = oracle.decode(qq, kc, vc, bt, sl, sc)
        for b in range(2):
            for h in range(2):
                np.testing.assert_allclose(out[b, h], Vc[b][:, h].astype(np.float64).mean(0),
                                           atol=1e-14)


def test_constant_v_rows_give_that_constant():
    rng = np.random.default_rng(6)
    lens = [25, 7]
    Kc = [rng.standard_normal((L, 1, 8)).astype(np.float32) for L in lens]
    c = rng.standard_normal(8).astype(np.float32)
    Vc = [np.broadcast_to(c, (L, 1, 8)).copy() for L in lens]
    q = rng.standard_normal((2, 3, 8)).astype(np.float32)
    kc, vc, bt, sl = paged_from_contiguous(Kc, Vc, 4)
    out = oracle.decode(q, kc, vc, bt, sl, 1.0)
    for b in range(2):
        for h in range(3):
            np.testing.assert_allclose(out[b, h], c.astype(np.float64), rtol=1e-14, atol=1e-15)


def test_zero_length_request_writes_zeros():
    q, Kc, Vc = rand_problem([5, 9], 2, 1, 8, seed=1)
    kc, vc, bt, sl = paged_from_contiguous(Kc, Vc, 4)
    sl = sl.copy()
    sl[0] = 0
    out = oracle.decode(q, kc, vc, bt, sl, 1.0)
    np.testing.assert_array_equal(out[0], 0.0)


def test_bf16_inputs_are_upcast_exactly():
    import workloads
    rng = np.random.default_rng(9)
    lens = [20, 3]
    Kc = [rng.standard_normal((L, 2, 16)).astype(np.float32) for L in lens]
    Vc = [rng.standard_normal((L, 2, 16)).astype(np.float32) for L in lens]
    q = rng.standard_normal((2, 4, 16)).astype(np.float32)
    Kb = [workloads.f32_to_bf16_bits(k) for k in Kc]
    Vb = [workloads.f32_to_bf16_bits(v) for v in Vc]
    qb = workloads.f32_to_bf16_bits(q)
    kc, vc, bt, sl = paged_from_contiguous(Kb, Vb, 8, dtype=np.uint16, fill=0x7FC0)
    out = oracle.decode(qb, kc, vc, bt, sl, 0.25)
    Kf = [brute.bf16_bits_to_f64(k) for k in Kb]
    Vf = [brute.bf16_bits_to_f64(v) for v in Vb]
    ref = brute_all(brute.bf16_bits_to_f64(qb), Kf, Vf, 0.25)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_out_of_range_table_entry_is_reported():
    q, Kc, Vc = rand_problem([5], 1, 1, 4, seed=1)
    kc, vc, bt, sl = paged_from_contiguous(Kc, Vc, 4)
    bt = bt.copy()
    bt[0, 1] = 999
    with pytest.raises(oracle.OracleError):
        oracle.decode(q, kc, vc, bt, sl, 1.0)


# ---------------------------------------------------------------------------
# write / copy / swap
# ---------------------------------------------------------------------------

def test_kv_cache_write_hand_example():
    NB, Hkv, bs, d = 3, 2, 4, 2
    kc = np.full((NB, Hkv, bs, d), np.nan, np.float32)
    vc = np.full((NB, Hkv, bs, d), np.nan, np.float32)
    k = np.arange(3 * Hkv * d, dtype=np.float32).reshape(3, Hkv, d)
    v = -k
    slots = np.array([9, -1, 2], np.int64)  # block 2 offset 1; skipped; block 0 offset 2
    bad = oracle.kv_cache_write(k, v, slots, kc, vc)
    assert bad == 0
    np.testing.assert_array_equal(kc[2, :, 1, :], k[0])
    np.testing.assert_array_equal(vc[2, :, 1, :], v[0])
    np.testing.assert_array_equal(kc[0, :, 2, :], k[2])
    written = np.zeros(kc.shape, bool)
    written[2, :, 1, :] = True
    written[0, :, 2, :] = True
    assert np.all(np.isnan(kc[~written])) and np.all(np.isnan(vc[~written]))
    assert oracle.kv_cache_write(k, v, np.array([12, 0, 0], np.int64), kc, vc) == 1


def test_kv_cache_write_bit_exact_on_nan_payloads():
    NB, Hkv, bs, d = 2, 1, 2, 4
    kc = np.zeros((NB, Hkv, bs, d), np.uint16)
    vc = np.zeros((NB, Hkv, bs, d), np.uint16)
    k = np.array([[[0x7FC1, 0xFFFF, 0x0001, 0x8000]]], np.uint16)
    oracle.kv_cache_write(k, k, np.array([3], np.int64), kc, vc)
    np.testing.assert_array_equal(kc[1, 0, 1], k[0, 0])


def test_copy_blocks_hand_example():
    NB, Hkv, bs, d = 4, 2, 2, 2
    kc = np.arange(NB * Hkv * bs * d, dtype=np.float32).reshape(NB, Hkv, bs, d)
    vc = -kc
    k0, v0 = kc.copy(), vc.copy()
    bad = oracle.copy_blocks(kc, vc, np.array([[1, 3], [0, 2]], np.int64))
    assert bad == 0
    np.testing.assert_array_equal(kc[3], k0[1])
    np.testing.assert_array_equal(kc[2], k0[0])
    np.testing.assert_array_equal(vc[3], v0[1])
    np.testing.assert_array_equal(kc[:2], k0[:2])
    assert oracle.copy_blocks(kc, vc, np.array([[0, 4]], np.int64)) == 1


def test_swap_blocks_hand_example():
    src = np.arange(3 * 1 * 2 * 2, dtype=np.float32).reshape(3, 1, 2, 2)
    dst = np.zeros((2, 1, 2, 2), np.float32)
    dv = np.zeros_like(dst)
    assert oracle.swap_blocks(src, -src, dst, dv, np.array([[2, 0], [0, 1]], np.int64)) == 0
    np.testing.assert_array_equal(dst[0], src[2])
    np.testing.assert_array_equal(dst[1], src[0])
    np.testing.assert_array_equal(dv[0], -src[2])


# ---------------------------------------------------------------------------
# fp8 e4m3
# ---------------------------------------------------------------------------

def _e4m3_value(c: int) -> float:
    """Value of an e4m3 code, straight from the format definition."""
    s = -1.0 if c & 0x80 else 1.0
    e = (c >> 3) & 0xF
    m = c & 7
    if e == 15 and m == 7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1 + m / 8.0) * 2.0 ** (e - 7)


def test_e4m3_decode_matches_torch_all_codes():
    torch = pytest.importorskip("torch")
    codes = np.arange(256, dtype=np.uint8)
    kc = codes.reshape(256, 1, 1, 1)
    # decode each code through the oracle: one 1-token request per code, q = 0
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([_e4m3_value(int(c)) for c in codes])
    np.testing.assert_array_equal(np.isnan(mine), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(mine[ok], ref[ok])
    # and through the oracle's decode path (V row of a length-1 request, scale 2)
    q = np.zeros((256, 1, 1), np.float32)
    bt = np.arange(256, dtype=np.int32).reshape(256, 1)
    sl = np.ones(256, np.int32)
    out = oracle.decode(q, kc, kc, bt, sl, 1.0, k_scale=np.array([2.0], np.float32),
                        v_scale=np.array([2.0], np.float32))
    got = out[:, 0, 0]
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    np.testing.assert_array_equal(got[ok], 2.0 * ref[ok])


def test_e4m3_quantize_known_values_and_nearest():
    vals = np.array([0.0, 1.0, -1.0, 448.0, 500.0, -1e9, 2.0 ** -9, 2.0 ** -10,
                     3 * 2.0 ** -10, 1.0625, 1.1875, 0.3], np.float32)
    codes = oracle.quantize_e4m3(vals, 1.0)
    assert codes[0] == 0x00 and codes[1] == 0x38 and codes[2] == 0xB8
    assert codes[3] == 0x7E and codes[4] == 0x7E and codes[5] == 0xFE
    assert codes[6] == 0x01          # smallest subnormal
    assert codes[7] == 0x00          # half of it: tie to even (zero)
    assert codes[8] == 0x02          # 1.5 x smallest: tie to even (2)
    assert codes[9] == 0x38          # 1.0625 halfway 1.0/1.125 -> even (1.0)
    assert codes[10] == 0x3A         # 1.1875 halfway 1.125/1.25 -> even (1.25)
    # nearest for random inputs, against a brute search over the code table
    x = np.random.default_rng(0).standard_normal(2000).astype(np.float32) * 30
    sc = np.float32(0.37)
    cq = oracle.quantize_e4m3(x, float(sc))
    table = np.array([_e4m3_value(c) for c in range(0x7F)])
    for xi, ci in zip(x, cq):
        y = float(np.float32(xi) / sc)
        a = min(abs(y), 448.0)
        best = np.min(np.abs(table - a))
        assert abs(abs(_e4m3_value(int(ci))) - a) == best
        assert (int(ci) & 0x80 != 0) == (y < 0)


def test_e4m3_quantize_matches_torch_in_range():
    torch = pytest.importorskip("torch")
    x = (np.random.default_rng(1).standard_normal(5000) * 50).astype(np.float32)
    x = np.clip(x, -440, 440)
    mine = oracle.quantize_e4m3(x, 1.0)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(mine, ref)


# ---------------------------------------------------------------------------
# figures printed on the pages
# ---------------------------------------------------------------------------

def _golden():
    path = os.path.join(os.path.dirname(__file__), "golden", "kv_sizing.txt")
    vals = {}
    for line in open(path):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = (s.strip() for s in line.split("="))
            vals[k] = float(v) if "." in v else int(v)
    return vals


def test_byte_model_reproduces_printed_size():
    g = _golden()
    n = byte_model.kv_cache_size_bytes(g["kv_cache_layers"], g["kv_cache_kv_heads"],
                                       g["kv_cache_head_dim"], g["kv_cache_seq_len"],
                                       g["kv_cache_batch"], g["kv_cache_bytes_per_value"])
    assert n == 8_589_934_592 == 2 ** 33
    assert f"{n / 1e9:.1f}" == f"{g['kv_cache_gb_printed']:.1f}"
    # one layer of that cache is the 4k x batch-16 decode workload's K+V bytes
    assert n // g["kv_cache_layers"] == 268_435_456
    assert byte_model.decode_algorithmic_bytes([4096] * 16, 32, 8, 128, 2, 2, 2) == \
        268_435_456 + 16 * 32 * 128 * 4


def test_waste_figures():
    g = _golden()
    assert byte_model.unused_slots_contiguous(200, 4096) == g["contiguous_waste_200_of_4096"]
    assert byte_model.unused_slots_paged(200, g["default_block_size"]) == 8
    worst = max(byte_model.unused_slots_paged(n, 16) for n in range(1, 1000))
    assert worst == g["paged_waste_bound_block16"]
    assert byte_model.unused_slots_paged(4096, 16) == 0


# ---------------------------------------------------------------------------
# planted mistakes: each must be caught by at least one pin
# ---------------------------------------------------------------------------

def _pin_suite(lib):
    """A compact run of the pins above against a given oracle build; returns
    the names of the pins that fail."""
    fails = []
    lens = [1, 9, 40, 77]
    q, Kc, Vc = rand_problem(lens, 4, 2, 16, seed=77)
    NB = 30
    kc, vc, bt, sl = paged_from_contiguous(Kc, Vc, 8, NB=NB,
                                           perm=np.random.default_rng(1).permutation(NB))
    try:
        got = oracle.decode(q, kc, vc, bt, sl, 0.25, lib=lib)
        if not np.allclose(got, brute_all(q, Kc, Vc, 0.25), rtol=0, atol=1e-12):
            fails.append("brute")
    except oracle.OracleError:
        fails.append("brute-error")
    try:
        w = oracle.decode_weights(q, kc, vc, bt, sl, 0.25, 3, 1, lib=lib)
        if abs(w.sum() - 1) > 1e-12 or len(w) != lens[3]:
            fails.append("weights")
    except oracle.OracleError:
        fails.append("weights-error")
    kk = np.full((4, 2, 4, 2), np.nan, np.float32)
    vv = kk.copy()
    k = np.arange(2 * 2 * 2, dtype=np.float32).reshape(2, 2, 2)
    oracle.kv_cache_write(k, k, np.array([9, 2], np.int64), kk, vv, lib=lib)
    if not (np.array_equal(kk[2, :, 1], k[0]) and np.array_equal(kk[0, :, 2], k[1])):
        fails.append("write")
    a = np.arange(4 * 2 * 2 * 2, dtype=np.float32).reshape(4, 2, 2, 2)
    a0 = a.copy()
    oracle.copy_blocks(a, a.copy(), np.array([[1, 3]], np.int64), lib=lib)
    if not np.array_equal(a[3], a0[1]):
        fails.append("copy")
    # the split-sequence restatement (partitions of 16 tokens over 8-token
    # blocks, so a partition's running max grows inside it) equals brute force
    try:
        got = oracle.decode_partitioned(q, kc, vc, bt, sl, 0.25, 16, lib=lib)
        if not np.allclose(got, brute_all(q, Kc, Vc, 0.25), rtol=0, atol=1e-12):
            fails.append("partitioned")
    except oracle.OracleError:
        fails.append("partitioned-error")
    # swap between pools of 3 and 2 blocks: dst[0] = src[1]
    src = np.arange(3 * 2 * 2 * 2, dtype=np.float32).reshape(3, 2, 2, 2)
    dst = np.zeros((2, 2, 2, 2), np.float32)
    dst_v = dst.copy()
    oracle.swap_blocks(src, src + 100, dst, dst_v, np.array([[1, 0]], np.int64), lib=lib)
    if not (np.array_equal(dst[0], src[1]) and np.array_equal(dst_v[0], src[1] + 100)
            and not dst[1].any()):
        fails.append("swap")
    # e4m3 codes fixed by the format (bias 7, 3 mantissa bits, subnormals below
    # 2^-6, largest finite 448) and round-to-nearest-even: 1, the two ties
    # next to it, saturation both ways, the smallest subnormal and a subnormal tie
    x = np.array([1.0, 1.0625, 1.1875, 1000.0, -1000.0, 2.0 ** -9, 1.5 * 2.0 ** -9],
                 np.float32)
    want = np.array([0x38, 0x38, 0x3A, 0x7E, 0xFE, 0x01, 0x02], np.uint8)
    if not np.array_equal(oracle.quantize_e4m3(x, 1.0, lib=lib), want):
        fails.append("e4m3")
    return fails


def test_pins_pass_on_the_real_oracle():
    assert _pin_suite(oracle.load()) == []


@pytest.mark.parametrize("mutant", list(range(1, 16)))
def test_planted_mistake_is_caught(mutant):
    with tempfile.TemporaryDirectory() as td:
        path = oracle.build(mutant=mutant, out_path=os.path.join(td, f"m{mutant}.so"))
        lib = oracle.load(path)
        assert _pin_suite(lib), f"mutant {mutant} slipped through every pin"
