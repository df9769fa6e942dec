"""Seeded random configurations against the oracle (GPU).

Each seed draws a batch (1..20 requests, lengths 0..3000), a head layout
(1..32 query heads per kv head), head_dim 64 or 128, a block size 1..256, the
cache type (fp32, bf16, or fp8 where the tensor-core path serves it), the
output type and the split (automatic or a fixed partition), runs fork-free
append + decode, and compares with the oracle: caches bit for bit, outputs
within the decode tolerance.  A second set draws prefix groups for the
prefix-aware decode."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workloads
from _helpers import DevWorkload, assert_decode_close, host_step, to_dev, to_host_bits, to_host_f64

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _draw(seed):
    rng = np.random.default_rng(9000 + seed)
    G = int(rng.choice([1, 2, 3, 4, 5, 8, 16, 32]))
    Hkv = int(rng.choice([1, 2, 4, 8])) if G <= 8 else int(rng.choice([1, 2]))
    d = int(rng.choice([64, 128]))
    bs = int(rng.choice([1, 2, 4, 8, 16, 16, 32, 64, 128, 256]))
    dtype = str(rng.choice(["f32", "bf16", "bf16", "fp8"]))
    if dtype == "fp8" and bs < 8:
        dtype = "bf16"
    B = int(rng.integers(1, 21))
    lens = [int(x) for x in rng.integers(0, 3001, size=B)]
    if rng.random() < 0.3:
        lens[int(rng.integers(0, B))] = 0
    part = int(rng.choice([0, 0, 64, 256, 1024]))
    out_f32 = bool(rng.random() < 0.5) or dtype == "f32"
    return dict(G=G, Hkv=Hkv, d=d, bs=bs, dtype=dtype, lens=lens, part=part, out_f32=out_f32)


@pytest.mark.parametrize("seed", range(60))
def test_random_configuration(seed):
    import paged_kv_cache_412_b200 as pkv
    c = _draw(seed)
    w = workloads.make_paged(c["lens"], Hq=c["G"] * c["Hkv"], Hkv=c["Hkv"], d=c["d"],
                             bs=c["bs"], dtype=c["dtype"], seed=9100 + seed, table_pad=2)
    kc, vc = host_step(w)
    ref = oracle.decode(w.q, kc, vc, w.block_tables, w.seq_lens, w.scale, k_scale=w.k_scale,
                        v_scale=w.v_scale)
    dw = DevWorkload(w)
    if w.slot_mapping.shape[0]:
        if c["dtype"] == "fp8":
            pkv.kv_cache_write_fp8(dw.k_new, dw.v_new, dw.slot_mapping, dw.k_cache, dw.v_cache,
                                   dw.k_scale, dw.v_scale)
        else:
            pkv.kv_cache_write(dw.k_new, dw.v_new, dw.slot_mapping, dw.k_cache, dw.v_cache)
    out_dtype = torch.float32 if c["out_f32"] else torch.bfloat16
    out = pkv.paged_attention_decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens,
                                     w.bs, w.scale, out_dtype=out_dtype,
                                     partition_size=c["part"], k_scale=dw.k_scale,
                                     v_scale=dw.v_scale)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0, c
    if c["dtype"] == "f32":
        assert np.array_equal(to_host_bits(dw.k_cache).view(np.uint32), kc.view(np.uint32)), c
    else:
        assert np.array_equal(to_host_bits(dw.k_cache), kc), c
    in_dt = "f32" if c["dtype"] == "f32" else "bf16"
    assert_decode_close(to_host_f64(out), ref, in_dt, "f32" if c["out_f32"] else "bf16",
                        what=str(c))


@pytest.mark.parametrize("seed", range(24))
def test_random_prefix_groups(seed):
    import paged_kv_cache_412_b200 as pkv
    rng = np.random.default_rng(9500 + seed)
    bs = int(rng.choice([8, 16, 32, 64, 128]))
    d = int(rng.choice([64, 128]))
    G = int(rng.choice([1, 2, 3, 4, 8, 16]))
    Hkv = int(rng.choice([1, 2, 4, 8])) if G <= 8 else 2
    ngroups = int(rng.integers(1, 4))
    groups = [(int(rng.integers(1, 24)), int(rng.integers(0, 40)) * bs) for _ in range(ngroups)]
    w = workloads.prefix_groups(groups, int(rng.integers(0, 4)), bs=bs, Hq=G * Hkv, Hkv=Hkv, d=d,
                                short_members=int(rng.integers(0, 3)), suffix_hi=600,
                                seed=9600 + seed)
    ref = oracle.decode(w.q, *host_step(w), w.block_tables, w.seq_lens, w.scale)
    dw = DevWorkload(w)
    if w.slot_mapping.shape[0]:
        pkv.kv_cache_write(dw.k_new, dw.v_new, dw.slot_mapping, dw.k_cache, dw.v_cache)
    out = pkv.paged_attention_decode_prefix(
        dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens,
        to_dev(w.info["prefix_of"]), to_dev(w.info["prefix_lens"]), w.bs, w.scale,
        out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0, groups
    assert_decode_close(to_host_f64(out), ref, "bf16", "f32", what=f"{groups} bs {bs} d {d} G {G}")
