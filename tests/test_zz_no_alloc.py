"""The decode entry point that allocates nothing (GPU).

Some callers cannot give this library a scratch buffer -- an engine that has
reserved nearly all device memory for its KV pool and forbids extensions to
allocate, or a latency-critical path that cannot afford cudaMalloc's
synchronisation.  pkv_paged_attention_decode_noalloc serves them from a fixed
scratch array inside the library.  These checks call it through the C ABI on
two calls in a row of different sizes (the shared array keeps the first call's
contents when the second one runs) and compare each result with the ordinary
entry point (which takes a workspace) and with the CPU oracle, within the
parity tolerances of the other decode tests.  This file is named so that
pytest collects it last.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workloads
from _helpers import DevWorkload, assert_decode_close, host_step, to_host_f64

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkv():
    import paged_kv_cache_412_b200 as m
    return m


def _check(pkv, w, partition_size=0, what=""):
    """Append, then decode through both entry points; compare each with the
    oracle and with each other."""
    dw = DevWorkload(w)
    fp8 = w.dtype == "fp8"
    if fp8:
        pkv.kv_cache_write_fp8(dw.k_new, dw.v_new, dw.slot_mapping, dw.k_cache, dw.v_cache,
                               dw.k_scale, dw.v_scale)
    else:
        pkv.kv_cache_write(dw.k_new, dw.v_new, dw.slot_mapping, dw.k_cache, dw.v_cache)
    kw = dict(out_dtype=torch.float32, partition_size=partition_size, k_scale=dw.k_scale,
              v_scale=dw.v_scale)
    ref_gpu = pkv.paged_attention_decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables,
                                         dw.seq_lens, w.bs, w.scale, **kw)
    got = pkv.paged_attention_decode_noalloc(dw.q, dw.k_cache, dw.v_cache, dw.block_tables,
                                             dw.seq_lens, w.bs, w.scale, **kw)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    kc, vc = host_step(w)
    ref = oracle.decode(w.q, kc, vc, w.block_tables, w.seq_lens, w.scale, k_scale=w.k_scale,
                        v_scale=w.v_scale)
    in_dt = "bf16" if w.dtype in ("bf16", "fp8") else "f32"
    got_h = to_host_f64(got)
    assert_decode_close(got_h, ref, in_dt, "f32", what=f"{what} vs oracle")
    assert_decode_close(got_h, to_host_f64(ref_gpu), in_dt, "f32",
                        what=f"{what} vs the workspace entry point")


def test_noalloc_matches_oracle_and_workspace_entry_point_two_calls(pkv):
    # first call: requests long enough to be split across CTAs (partial records)
    w1 = workloads.make_paged([3000, 700, 1, 4096], Hq=32, Hkv=8, d=128, bs=16, dtype="bf16",
                              seed=41)
    _check(pkv, w1, what="no-alloc call 1")
    # second call, other sizes and a fixed split, reusing the same scratch array
    w2 = workloads.make_paged([50, 900, 2000], Hq=16, Hkv=2, d=64, bs=8, dtype="bf16", seed=42)
    _check(pkv, w2, partition_size=256, what="no-alloc call 2")


def test_noalloc_fp8_cache_forwards_scales(pkv):
    w = workloads.make_paged([1500, 33, 2600], Hq=32, Hkv=8, d=128, bs=16, dtype="fp8", seed=43)
    _check(pkv, w, what="no-alloc fp8")


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
    # an argument error is reported as such, whatever the size
    with pytest.raises(pkv.PkvError) as ei:
        pkv.paged_attention_decode_noalloc(q, kc, kc, bt, sl, 16, float("nan"), max_seq_len=4096)
    assert ei.value.status == 1
