"""fp8 (e4m3) KV cache on the GPU: quantising append and decode.

"KV Cache Management" ("Watch Out For", "What to Read Next"): long contexts
call for an 8-bit KV cache.  The append must produce exactly the oracle's e4m3
codes (round to nearest even of the fp32 quotient x / scale, saturating);
decode reads code * scale and must match the oracle's fp64 attention over the
same codes within the bf16 tolerances."""
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


def _step(pkv, dw, out_dtype=None, partition_size=0):
    w = dw.w
    if w.copy_pairs.shape[0]:
        pkv.copy_blocks(dw.k_cache, dw.v_cache, dw.copy_pairs)
    if w.slot_mapping.shape[0]:
        pkv.kv_cache_write_fp8(dw.k_new, dw.v_new, dw.slot_mapping, dw.k_cache, dw.v_cache,
                               dw.k_scale, dw.v_scale)
    out = pkv.paged_attention_decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens,
                                     w.bs, w.scale, out_dtype=out_dtype,
                                     partition_size=partition_size, k_scale=dw.k_scale,
                                     v_scale=dw.v_scale)
    torch.cuda.synchronize()
    return out


def test_quantising_append_is_bit_exact(pkv):
    rng = np.random.default_rng(5)
    NB, Hkv, bs, d, T = 32, 4, 16, 128, 200
    k = workloads.f32_to_bf16_bits(rng.standard_normal((T, Hkv, d), dtype=np.float32) * 40)
    v = workloads.f32_to_bf16_bits(rng.standard_normal((T, Hkv, d), dtype=np.float32))
    ks = np.array([0.01, 0.1, 1.0, 0.37], np.float32)  # 40-sigma / 0.01 saturates at 448
    vs = np.array([0.5, 0.02, 0.003, 2.0], np.float32)
    slots = rng.permutation(NB * bs)[:T].astype(np.int64)
    slots[3] = -1
    kc = np.full((NB, Hkv, bs, d), workloads.E4M3_NAN, np.uint8)
    vc = kc.copy()
    from _helpers import quantize_tokens
    kref, vref = kc.copy(), vc.copy()
    oracle.kv_cache_write(quantize_tokens(k, ks), quantize_tokens(v, vs), slots, kref, vref)
    dk, dv = to_dev(kc), to_dev(vc)
    pkv.kv_cache_write_fp8(to_dev(k), to_dev(v), to_dev(slots), dk, dv, to_dev(ks), to_dev(vs))
    torch.cuda.synchronize()
    assert np.array_equal(dk.cpu().numpy(), kref)
    assert np.array_equal(dv.cpu().numpy(), vref)


CASES = [
    ([1, 17, 100, 200], 32, 8, 128, 16),
    ([513, 64, 65, 3000], 8, 1, 128, 8),     # G = 8, block 8
    ([90, 700], 32, 2, 128, 64),             # G = 16, block = stage
    ([300, 129, 2], 8, 4, 64, 32),           # d 64
    ([0, 40, 1], 4, 2, 128, 256),            # empty request, block > stage
    ([50, 1, 333], 8, 8, 128, 16),           # G = 1
    ([200, 77], 12, 4, 128, 16),             # G = 3 (padded to 8)
    ([120, 260], 32, 1, 64, 16),             # G = 32 at d 64: two 16-head passes per kv head
    ([1000, 3], 16, 1, 64, 128),             # G = 16, d 64, block 128
    # 60 requests of 1..400 tokens: many segments per CTA, split across the consumers
    ([int(x) for x in np.random.default_rng(77).integers(1, 401, size=60)], 32, 8, 128, 16),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"L{len(c[0])}_G{c[1]//c[2]}_d{c[3]}_bs{c[4]}")
def test_fp8_step_parity(pkv, case):
    lens, Hq, Hkv, d, bs = case
    w = workloads.make_paged(lens, Hq=Hq, Hkv=Hkv, d=d, bs=bs, dtype="fp8",
                             seed=2000 + sum(lens) + bs, pool_factor=1.2, extra_blocks=2,
                             table_pad=1)
    kc_ref, vc_ref = host_step(w)
    ref = oracle.decode(w.q, kc_ref, vc_ref, w.block_tables, w.seq_lens, w.scale,
                        k_scale=w.k_scale, v_scale=w.v_scale)
    for out_dtype in (None, torch.float32):
        dw = DevWorkload(w)
        out = _step(pkv, dw, out_dtype=out_dtype)
        assert np.array_equal(to_host_bits(dw.k_cache), kc_ref)
        assert np.array_equal(to_host_bits(dw.v_cache), vc_ref)
        od = "f32" if out_dtype == torch.float32 else "bf16"
        assert_decode_close(to_host_f64(out), ref, "bf16", od, what=f"fp8 {case} {od}")
    assert pkv.get_device_error() == 0


def test_fp8_fixed_partitions(pkv):
    w = workloads.make_paged([3000, 257, 1], Hq=16, Hkv=2, d=128, bs=16, dtype="fp8", seed=8)
    kc_ref, vc_ref = host_step(w)
    ref = oracle.decode(w.q, kc_ref, vc_ref, w.block_tables, w.seq_lens, w.scale,
                        k_scale=w.k_scale, v_scale=w.v_scale)
    dw = DevWorkload(w)
    _step(pkv, dw)
    for P in (64, 192, 1024):
        out = pkv.paged_attention_decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables,
                                         dw.seq_lens, w.bs, w.scale, partition_size=P,
                                         k_scale=dw.k_scale, v_scale=dw.v_scale,
                                         out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert_decode_close(to_host_f64(out), ref, "bf16", "f32", what=f"fp8 P={P}")


def test_workload_gqa_4k_fp8(pkv):
    w = workloads.gqa_4k_fp8()
    kc_ref, vc_ref = host_step(w)
    dw = DevWorkload(w)
    out = _step(pkv, dw, out_dtype=torch.float32)
    assert np.array_equal(to_host_bits(dw.k_cache), kc_ref)
    rows = [0, 5, 15]
    ref = oracle.decode(w.q[rows], kc_ref, vc_ref, w.block_tables[rows], w.seq_lens[rows], w.scale,
                        k_scale=w.k_scale, v_scale=w.v_scale)
    assert_decode_close(to_host_f64(out)[rows], ref, "bf16", "f32", what="gqa_4k fp8")
    assert pkv.get_device_error() == 0


def test_fp8_needs_scales_and_tensor_core_block_sizes(pkv):
    w = workloads.make_paged([40], Hq=4, Hkv=2, d=128, bs=16, dtype="fp8", seed=1)
    dw = DevWorkload(w)
    with pytest.raises(pkv.PkvError) as ei:
        pkv.paged_attention_decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens,
                                   w.bs, w.scale)
    assert ei.value.status == 1
