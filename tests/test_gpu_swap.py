"""Block swap between the device cache and a pinned host pool (GPU).

Preemption ("PagedAttention: Optimizing KV Cache Utilization in Large Language
Models", "Conclusion"): a request's blocks are swapped out to host memory and
later swapped back in, possibly into other physical blocks.  Both directions
must be bit-exact against the oracle's pool-to-pool copy; pointers the device
cannot reach are refused without a launch."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workloads
from _helpers import to_dev, to_host_bits

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkv():
    import paged_kv_cache_412_b200 as m
    return m


def _pinned(a: np.ndarray):
    t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
    t = t.pin_memory()
    return t.view(torch.bfloat16) if a.dtype == np.uint16 else t


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_swap_out_and_in_bit_exact(pkv, dtype):
    w = workloads.make_paged([300, 77, 1000], Hq=8, Hkv=4, d=128, bs=16, dtype=dtype, seed=9,
                             extra_blocks=10, append_last=False)
    nb_host = 128
    host_k = np.full((nb_host,) + w.k_cache.shape[1:], 0, w.k_cache.dtype)
    host_v = host_k.copy()
    pairs_out = np.stack([w.block_tables[2, :40].astype(np.int64),
                          np.arange(5, 45, dtype=np.int64)], axis=1)
    # swap out: device cache -> pinned host pool (mapping in device memory)
    dk, dv = to_dev(w.k_cache), to_dev(w.v_cache)
    hk, hv = _pinned(host_k), _pinned(host_v)
    pkv.swap_blocks(dk, dv, hk, hv, to_dev(pairs_out))
    torch.cuda.synchronize()
    assert oracle.swap_blocks(w.k_cache, w.v_cache, host_k, host_v, pairs_out) == 0
    got = hk.view(torch.int16).numpy().view(np.uint16) if dtype == "bf16" else hk.numpy()
    assert np.array_equal(got.view(np.uint8), host_k.view(np.uint8))
    # swap in: host pool -> other device blocks (mapping in pinned host memory)
    pairs_in = np.stack([np.arange(5, 45, dtype=np.int64),
                         np.arange(w.num_blocks - 40, w.num_blocks, dtype=np.int64)], axis=1)
    kc_ref, vc_ref = w.k_cache.copy(), w.v_cache.copy()
    assert oracle.swap_blocks(host_k, host_v, kc_ref, vc_ref, pairs_in) == 0
    pkv.swap_blocks(hk, hv, dk, dv, torch.from_numpy(pairs_in).pin_memory(), device=0)
    torch.cuda.synchronize()
    assert np.array_equal(to_host_bits(dk).view(np.uint8), kc_ref.view(np.uint8))
    assert np.array_equal(to_host_bits(dv).view(np.uint8), vc_ref.view(np.uint8))
    assert pkv.get_device_error() == 0


def test_bad_pair_flagged_and_unreachable_memory_refused(pkv):
    w = workloads.make_paged([64], Hq=4, Hkv=2, d=64, bs=16, dtype="bf16", seed=3,
                             append_last=False)
    dk, dv = to_dev(w.k_cache), to_dev(w.v_cache)
    hk = _pinned(np.zeros((8,) + w.k_cache.shape[1:], np.uint16))
    hv = _pinned(np.zeros((8,) + w.k_cache.shape[1:], np.uint16))
    pairs = to_dev(np.array([[0, 1], [1, 99]], np.int64))
    pkv.swap_blocks(dk, dv, hk, hv, pairs)
    assert pkv.get_device_error() & pkv.DEVERR["BAD_PAIR"]
    # pageable host memory is not reachable from the device: refused, nothing runs
    L = pkv._get_lib()
    pageable = np.zeros((8,) + w.k_cache.shape[1:], np.uint16)
    import ctypes
    st = L.pkv_swap_blocks(ctypes.c_void_p(dk.data_ptr()), ctypes.c_void_p(dv.data_ptr()),
                           ctypes.c_void_p(pageable.ctypes.data),
                           ctypes.c_void_p(pageable.ctypes.data),
                           ctypes.c_void_p(pairs.data_ptr()), 1, w.num_blocks, 8, 2, 64, 16, 1,
                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 1
    assert pkv.get_device_error() == 0
