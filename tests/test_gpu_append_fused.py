"""GPU parity of paged_attention_decode_append: the append of each request's
new token fused into the decode kernel.

PagedAttention ("The Mechanics of PagedAttention"): the step's new K and V rows
go to the slot the request's block table names for position L - 1, then the
decode reads the whole context.  The fused call must leave the caches bit-exact
equal to the oracle's kv_cache_write (NaN-poisoned slots nobody owns
untouched), give the decode the oracle's result within the bf16 bars, and give
bit-for-bit the same output as kv_cache_write followed by
paged_attention_decode (the same kernel, the same grid)."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workloads
from _helpers import (DevWorkload, assert_decode_close, host_step, to_dev, to_host_bits,
                      to_host_f64)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkv():
    import paged_kv_cache_412_b200 as m
    return m


def per_request_rows(w, x):
    """The workload's appended rows [T, Hkv, d] as one row per request
    [B, Hkv, d]; a request with no new token (length 0) gets a NaN row that
    must never reach the cache."""
    out = np.full((w.B, w.Hkv, w.d), workloads.BF16_NAN, dtype=np.uint16)
    rows = [b for b in range(w.B) if w.seq_lens[b] > 0]
    out[rows] = x
    return out


def fused(pkv, dw, w, out_dtype=None, partition_size=0):
    kn = to_dev(per_request_rows(w, w.k_new))
    vn = to_dev(per_request_rows(w, w.v_new))
    out = pkv.paged_attention_decode_append(dw.q, kn, vn, dw.k_cache, dw.v_cache,
                                            dw.block_tables, dw.seq_lens, w.bs, w.scale,
                                            out_dtype=out_dtype, partition_size=partition_size)
    torch.cuda.synchronize()
    return out


def separate(pkv, dw, w, out_dtype=None, partition_size=0):
    if w.slot_mapping.shape[0]:
        pkv.kv_cache_write(dw.k_new, dw.v_new, dw.slot_mapping, dw.k_cache, dw.v_cache)
    out = pkv.paged_attention_decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens,
                                     w.bs, w.scale, out_dtype=out_dtype,
                                     partition_size=partition_size)
    torch.cuda.synchronize()
    return out


def check_caches(dw, kc_ref, vc_ref):
    assert np.array_equal(to_host_bits(dw.k_cache), kc_ref), "k_cache differs"
    assert np.array_equal(to_host_bits(dw.v_cache), vc_ref), "v_cache differs"


CASES = [
    # lens, Hq, Hkv, d, bs
    ([33, 64, 65, 7, 1, 300], 8, 8, 128, 16),
    ([129, 31, 512], 32, 8, 128, 16),
    ([250, 3, 40], 16, 2, 128, 8),
    ([77, 160], 12, 4, 64, 32),
    ([90, 45], 16, 1, 128, 16),                   # G = 16
    ([70, 200, 5], 10, 2, 128, 4),                # row copies of 4-row blocks
    ([70, 200, 5, 64], 8, 2, 128, 2),             # row copies of 2-row blocks
    ([130, 1, 64], 16, 1, 64, 4),                 # d 64, G = 16, block size 4
    ([130, 1, 64, 700], 8, 2, 64, 4),             # d 64, G = 4, block size 4, in launch
    ([257, 33, 900], 16, 2, 64, 2),               # d 64, G = 8, block size 2, in launch
    ([300, 129], 8, 2, 128, 64),
    ([700, 129], 32, 8, 128, 128),                # block larger than a chunk
    ([513, 20, 300], 8, 4, 64, 256),
    ([0, 40, 0, 1], 4, 2, 128, 16),               # empty requests append nothing
    ([64, 65, 63, 128, 1], 8, 2, 64, 8),          # new token first / last in a chunk
    ([int(x) for x in np.random.default_rng(78).integers(1, 401, size=60)], 32, 8, 128, 16),
    # more (request, head group) pairs than four per SM: two CTAs per SM
    ([int(x) for x in np.random.default_rng(80).integers(1, 300, size=100)], 32, 8, 128, 8),
    ([int(x) for x in np.random.default_rng(81).integers(1, 300, size=100)], 32, 8, 128, 4),
    ([int(x) for x in np.random.default_rng(82).integers(1, 200, size=100)], 16, 8, 64, 2),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"L{len(c[0])}_G{c[1]//c[2]}_d{c[3]}_bs{c[4]}")
def test_fused_append_matches_oracle_and_separate_calls(pkv, case):
    lens, Hq, Hkv, d, bs = case
    w = workloads.make_paged(lens, Hq=Hq, Hkv=Hkv, d=d, bs=bs, dtype="bf16",
                             seed=2000 + sum(lens) + bs, pool_factor=1.3, extra_blocks=3,
                             table_pad=1)
    kc_ref, vc_ref = host_step(w)
    ref = oracle.decode(w.q, kc_ref, vc_ref, w.block_tables, w.seq_lens, w.scale)
    for out_dtype, od in ((None, "bf16"), (torch.float32, "f32")):
        dw = DevWorkload(w)
        out = fused(pkv, dw, w, out_dtype=out_dtype)
        assert pkv.get_device_error() == 0
        check_caches(dw, kc_ref, vc_ref)
        assert_decode_close(to_host_f64(out), ref, "bf16", od, what=f"{case} out={od}")
        dw2 = DevWorkload(w)
        out2 = separate(pkv, dw2, w, out_dtype=out_dtype)
        assert torch.equal(out.view(torch.int16) if od == "bf16" else out.view(torch.int32),
                           out2.view(torch.int16) if od == "bf16" else out2.view(torch.int32))


@pytest.mark.parametrize("P", [64, 512])
def test_fused_append_fixed_partitions(pkv, P):
    w = workloads.make_paged([1000, 33, 400, 1], Hq=8, Hkv=2, d=128, bs=16, dtype="bf16",
                             seed=77)
    kc_ref, vc_ref = host_step(w)
    ref = oracle.decode(w.q, kc_ref, vc_ref, w.block_tables, w.seq_lens, w.scale)
    dw = DevWorkload(w)
    out = fused(pkv, dw, w, partition_size=P)
    check_caches(dw, kc_ref, vc_ref)
    assert_decode_close(to_host_f64(out), ref, "bf16", "bf16", what=f"P={P}")


def test_fused_append_gqa_4k_full_size(pkv):
    """The 4k-context GQA workload (16 requests x 4096 tokens, 32 q / 8 kv
    heads, d 128, blocks of 16) at full size, as the benchmark step calls it."""
    w = workloads.gqa_4k()
    kc_ref, vc_ref = host_step(w)
    dw = DevWorkload(w)
    out = fused(pkv, dw, w)
    assert pkv.get_device_error() == 0
    check_caches(dw, kc_ref, vc_ref)
    rows = [0, 7, 15]
    ref = oracle.decode(w.q[rows], kc_ref, vc_ref, w.block_tables[rows], w.seq_lens[rows],
                        w.scale)
    assert_decode_close(to_host_f64(out)[rows], ref, "bf16", "bf16", what="gqa_4k fused")


def test_length_one_returns_new_v_row(pkv):
    """A request of one token attends only to the token it appends: the output
    is that token's V row, exactly (fp32 output)."""
    w = workloads.make_paged([1, 1, 1], Hq=8, Hkv=2, d=128, bs=16, dtype="bf16", seed=5)
    dw = DevWorkload(w)
    got = to_host_f64(fused(pkv, dw, w, out_dtype=torch.float32))
    vnew = workloads.bf16_bits_to_f32(w.v_new).astype(np.float64)
    for b in range(3):
        for h in range(8):
            np.testing.assert_array_equal(got[b, h], vnew[b, h // 4])


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (32, 2)], ids=["in_launch", "append_kernel"])
def test_fused_append_in_cuda_graph(pkv, Hq, Hkv):
    """Captured once, replayed twice: the append writes the same rows again
    and the output is unchanged.  8-head groups append inside the decode
    launch; 16-head groups through the append kernel launched before it."""
    w = workloads.make_paged([300, 17, 1000], Hq=Hq, Hkv=Hkv, d=128, bs=16, dtype="bf16", seed=11)
    kc_ref, vc_ref = host_step(w)
    ref = oracle.decode(w.q, kc_ref, vc_ref, w.block_tables, w.seq_lens, w.scale)
    dw = DevWorkload(w)
    kn = to_dev(per_request_rows(w, w.k_new))
    vn = to_dev(per_request_rows(w, w.v_new))
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.bfloat16, device="cuda")
    ws = pkv.new_workspace(pkv.decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.d, w.bs,
                                                      w.max_blocks * w.bs))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        pkv.paged_attention_decode_append(dw.q, kn, vn, dw.k_cache, dw.v_cache, dw.block_tables,
                                          dw.seq_lens, w.bs, w.scale, out, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        pkv.paged_attention_decode_append(dw.q, kn, vn, dw.k_cache, dw.v_cache, dw.block_tables,
                                          dw.seq_lens, w.bs, w.scale, out, workspace=ws)
    first = None
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize()
        check_caches(dw, kc_ref, vc_ref)
        assert_decode_close(to_host_f64(out), ref, "bf16", "bf16", what="graph replay")
        if first is None:
            first = out.clone()
        else:
            assert torch.equal(first.view(torch.int16), out.view(torch.int16))
    del g
    assert pkv.get_device_error() == 0


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (16, 1)], ids=["in_launch", "append_kernel"])
def test_new_token_in_bad_block_is_skipped_and_flagged(pkv, Hq, Hkv):
    """The new token's table entry outside the pool: nothing is written
    anywhere (the caches stay as they were) and PKV_DEVERR_BAD_BLOCK is set.
    8-head groups append inside the decode launch; 16-head groups through the
    separate append kernel."""
    w = workloads.make_paged([100, 40], Hq=Hq, Hkv=Hkv, d=128, bs=16, dtype="bf16", seed=21)
    bt = w.block_tables.copy()
    bt[1, (40 - 1) // 16] = w.num_blocks + 5
    dw = DevWorkload(w)
    dw.block_tables = to_dev(bt)
    fused(pkv, dw, w)
    assert pkv.get_device_error() & pkv.DEVERR["BAD_BLOCK"]
    # request 0's token is written, request 1's is not
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    assert oracle.kv_cache_write(w.k_new[:1], w.v_new[:1], w.slot_mapping[:1], kc, vc) == 0
    check_caches(dw, kc, vc)


def test_unsupported_and_invalid_arguments(pkv):
    w = workloads.make_paged([40, 9], Hq=8, Hkv=2, d=128, bs=16, dtype="bf16", seed=23)
    dw = DevWorkload(w)
    kn = to_dev(per_request_rows(w, w.k_new))
    vn = to_dev(per_request_rows(w, w.v_new))
    before = to_host_bits(dw.k_cache)
    # a k_new that does not start on a 16-byte boundary
    flat = torch.empty(kn.numel() + 1, dtype=torch.bfloat16, device="cuda")
    kn_odd = flat[1:].view(kn.shape)
    kn_odd.copy_(kn)
    with pytest.raises(pkv.PkvError, match="INVALID_ARG"):
        pkv.paged_attention_decode_append(dw.q, kn_odd, vn, dw.k_cache, dw.v_cache,
                                          dw.block_tables, dw.seq_lens, w.bs, w.scale)
    # block size 1 has no tensor-core path
    w1 = workloads.make_paged([40, 9], Hq=8, Hkv=2, d=128, bs=1, dtype="bf16", seed=23)
    dw1 = DevWorkload(w1)
    with pytest.raises(pkv.PkvError, match="UNSUPPORTED"):
        pkv.paged_attention_decode_append(dw1.q, kn, vn, dw1.k_cache, dw1.v_cache,
                                          dw1.block_tables, dw1.seq_lens, 1, w1.scale)
    # fp32 caches are refused by the binding before the call
    with pytest.raises(TypeError):
        pkv.paged_attention_decode_append(dw.q, kn, vn, dw.k_cache.float(), dw.v_cache.float(),
                                          dw.block_tables, dw.seq_lens, w.bs, w.scale)
    torch.cuda.synchronize()
    assert np.array_equal(to_host_bits(dw.k_cache), before)
    assert pkv.get_device_error() == 0
