"""The calls are capturable in a CUDA graph (GPU): a serving loop captures its
decode step once and replays it.  Each case captures fork + append + decode
(with an explicit workspace: nothing may allocate or synchronise inside a
capture), replays the graph, and compares with the oracle."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workloads
from _helpers import DevWorkload, assert_decode_close, host_step, to_dev, to_host_bits, to_host_f64

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _replay(fn, times=2):
    fn()  # eager first: per-device setup (occupancy, tensor-map encoder) happens outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    for _ in range(times):
        g.replay()
    torch.cuda.synchronize()
    return g


def test_step_graph_with_forks():
    import paged_kv_cache_412_b200 as pkv
    w = workloads.prefix_shared(poison=True, batch=12, suffix_lo=16, suffix_hi=80)
    kc_ref, vc_ref = host_step(w)
    ref = oracle.decode(w.q, kc_ref, vc_ref, w.block_tables, w.seq_lens, w.scale)
    dw = DevWorkload(w)
    L = int(w.seq_lens.max())
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    ws = pkv.new_workspace(pkv.decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.d, w.bs, L, 0))

    def step():
        pkv.copy_blocks(dw.k_cache, dw.v_cache, dw.copy_pairs)
        pkv.kv_cache_write(dw.k_new, dw.v_new, dw.slot_mapping, dw.k_cache, dw.v_cache)
        pkv.paged_attention_decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens,
                                   w.bs, w.scale, out, max_seq_len=L, workspace=ws)
    _replay(step)
    assert np.array_equal(to_host_bits(dw.k_cache), kc_ref)
    assert np.array_equal(to_host_bits(dw.v_cache), vc_ref)
    assert_decode_close(to_host_f64(out), ref, "bf16", "f32", what="graph step")
    assert pkv.get_device_error() == 0


def test_prefix_decode_graph():
    import paged_kv_cache_412_b200 as pkv
    w = workloads.prefix_groups([(9, 512), (4, 128)], 3, bs=16, Hq=32, Hkv=8, d=128, seed=1301)
    ref = oracle.decode(w.q, *host_step(w), w.block_tables, w.seq_lens, w.scale)
    dw = DevWorkload(w)
    L = int(w.seq_lens.max())
    po = to_dev(w.info["prefix_of"])
    pl = to_dev(w.info["prefix_lens"])
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    ws = pkv.new_workspace(pkv.decode_prefix_workspace_bytes(w.B, w.Hq, w.Hkv, w.d, w.bs, L,
                                                             len(w.info["prefix_lens"]), w.B, L))

    def step():
        pkv.kv_cache_write(dw.k_new, dw.v_new, dw.slot_mapping, dw.k_cache, dw.v_cache)
        pkv.paged_attention_decode_prefix(dw.q, dw.k_cache, dw.v_cache, dw.block_tables,
                                          dw.seq_lens, po, pl, w.bs, w.scale, out,
                                          max_seq_len=L, max_prefix_members=w.B,
                                          max_prefix_len=L, workspace=ws)
    _replay(step)
    assert_decode_close(to_host_f64(out), ref, "bf16", "f32", what="prefix graph")
    assert pkv.get_device_error() == 0


def test_fp8_step_graph():
    import paged_kv_cache_412_b200 as pkv
    w = workloads.make_paged([700, 1, 64, 1500], Hq=32, Hkv=8, d=128, bs=16, dtype="fp8",
                             seed=1302)
    kc_ref, vc_ref = host_step(w)
    ref = oracle.decode(w.q, kc_ref, vc_ref, w.block_tables, w.seq_lens, w.scale,
                        k_scale=w.k_scale, v_scale=w.v_scale)
    dw = DevWorkload(w)
    L = int(w.seq_lens.max())
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    ws = pkv.new_workspace(pkv.decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.d, w.bs, L, 0))

    def step():
        pkv.kv_cache_write_fp8(dw.k_new, dw.v_new, dw.slot_mapping, dw.k_cache, dw.v_cache,
                               dw.k_scale, dw.v_scale)
        pkv.paged_attention_decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.seq_lens,
                                   w.bs, w.scale, out, max_seq_len=L, workspace=ws,
                                   k_scale=dw.k_scale, v_scale=dw.v_scale)
    _replay(step)
    assert np.array_equal(to_host_bits(dw.k_cache), kc_ref)
    assert_decode_close(to_host_f64(out), ref, "bf16", "f32", what="fp8 graph")
    assert pkv.get_device_error() == 0
