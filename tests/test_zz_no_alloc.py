"""The decode entry point that allocates nothing (GPU).

Some callers cannot give this library a scratch buffer -- an engine that has
reserved nearly all device memory for its KV pool and forbids extensions to
allocate, or a latency-critical path that cannot afford cudaMalloc's
synchronisation.  pkv_paged_attention_decode_noalloc serves them from a fixed
scratch array inside the library.  These checks call it through the C ABI and
compare it with the ordinary entry point (which takes a workspace) on the same
inputs, on two calls in a row of different sizes (the shared array keeps the
first call's contents when the second one runs).  This file is named so that
pytest collects it last.
"""
from __future__ import annotations

import numpy as np
import pytest

import workloads
from _helpers import DevWorkload, assert_decode_close, to_host_f64

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkv():
    import paged_kv_cache_412_b200 as m
    return m


def _pair(pkv, w, partition_size=0):
    dw = DevWorkload(w)
    pkv.kv_cache_write(dw.k_new, dw.v_new, dw.slot_mapping, dw.k_cache, dw.v_cache)
    ref = pkv.paged_attention_decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens,
                                     w.bs, w.scale, out_dtype=torch.float32,
                                     partition_size=partition_size)
    got = pkv.paged_attention_decode_noalloc(dw.q, dw.k_cache, dw.v_cache, dw.block_tables,
                                             dw.seq_lens, w.bs, w.scale,
                                             out_dtype=torch.float32,
                                             partition_size=partition_size)
    torch.cuda.synchronize()
    return to_host_f64(got), to_host_f64(ref)


def test_noalloc_matches_workspace_entry_point_two_calls(pkv):
    # first call: requests long enough to be split across CTAs (partial records)
    w1 = workloads.make_paged([3000, 700, 1, 4096], Hq=32, Hkv=8, d=128, bs=16, dtype="bf16",
                              seed=41)
    got, ref = _pair(pkv, w1)
    assert_decode_close(got, ref, "bf16", "f32", what="no-alloc call 1")
    # second call, other sizes and a fixed split, reusing the same scratch array
    w2 = workloads.make_paged([50, 900, 2000], Hq=16, Hkv=2, d=64, bs=8, dtype="bf16", seed=42)
    got, ref = _pair(pkv, w2, partition_size=256)
    assert_decode_close(got, ref, "bf16", "f32", what="no-alloc call 2")
    assert pkv.get_device_error() == 0


def test_noalloc_refuses_sizes_beyond_its_scratch(pkv):
    cap = int(pkv._get_lib().pkv_decode_noalloc_scratch_bytes())
    # find a batch whose workspace exceeds the fixed array
    B = 16
    while pkv.decode_workspace_bytes(B, 32, 8, 128, 16, 4096, 0) <= cap:
        B *= 2
    q = torch.zeros((B, 32, 128), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((4, 8, 16, 128), dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros((B, 256), dtype=torch.int32, device="cuda")
    sl = torch.ones((B,), dtype=torch.int32, device="cuda")
    with pytest.raises(pkv.PkvError) as ei:
        pkv.paged_attention_decode_noalloc(q, kc, kc, bt, sl, 16, 0.1, max_seq_len=4096)
    assert ei.value.status == 3
