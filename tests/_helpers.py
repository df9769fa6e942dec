"""Shared test helpers: moving workloads to the device and the parity bars.

Tolerances (floating point; integer/byte work is compared bit-exactly):
* bf16 output: |gpu - oracle| <= 2e-3 + 1e-2 |oracle| per element (the
  max-abs 2e-3 / relative 1e-2 bar read in allclose form, because half an ulp
  of bf16 at |x| in [1, 2) is 3.9e-3, above 2e-3 on its own);
* fp32 output from bf16 inputs: |gpu - oracle| <= 2e-3 (isolates the fp32
  accumulation path from output rounding);
* fp32 inputs and output: |gpu - oracle| <= 1e-5 + 1e-5 |oracle|.
"""
from __future__ import annotations

import numpy as np

BF16_ABS, BF16_REL = 2e-3, 1e-2
F32OUT_ABS = 2e-3
F32_ABS, F32_REL = 1e-5, 1e-5


def to_dev(arr: np.ndarray, device="cuda"):
    import torch
    arr = np.ascontiguousarray(arr)
    if arr.dtype == np.uint16:  # bf16 bit patterns
        return torch.from_numpy(arr.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(arr).to(device)


def to_host_bits(t) -> np.ndarray:
    """Device tensor -> numpy with bf16 kept as uint16 bit patterns."""
    import torch
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def to_host_f64(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def decode_tolerance(ref: np.ndarray, in_dtype: str, out_dtype: str) -> np.ndarray:
    if in_dtype == "f32":
        return F32_ABS + F32_REL * np.abs(ref)
    if out_dtype == "bf16":
        return BF16_ABS + BF16_REL * np.abs(ref)
    return np.full(ref.shape, F32OUT_ABS)


def assert_decode_close(got: np.ndarray, ref: np.ndarray, in_dtype: str, out_dtype: str,
                        what: str = "") -> dict:
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    tol = decode_tolerance(ref, in_dtype, out_dtype)
    bad = err > tol
    stats = {"max_abs": float(err.max(initial=0.0)),
             "max_rel": float((err / np.maximum(np.abs(ref), 1e-30)).max(initial=0.0))}
    if bad.any():
        idx = np.argwhere(bad)[0]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} outputs out of tolerance; first at "
            f"{tuple(int(i) for i in idx)}: got {got[tuple(idx)]!r} ref {ref[tuple(idx)]!r}; "
            f"max_abs {stats['max_abs']:.3e}")
    return stats


class DevWorkload:
    """A workload's arrays on the device (torch tensors)."""

    def __init__(self, w, device="cuda"):
        import torch
        self.w = w
        self.q = to_dev(w.q, device)
        self.k_cache = to_dev(w.k_cache, device)
        self.v_cache = to_dev(w.v_cache, device)
        self.block_tables = to_dev(w.block_tables, device)
        self.seq_lens = to_dev(w.seq_lens, device)
        self.k_new = to_dev(w.k_new, device)
        self.v_new = to_dev(w.v_new, device)
        self.slot_mapping = to_dev(w.slot_mapping.astype(np.int64), device)
        self.copy_pairs = to_dev(w.copy_pairs.astype(np.int64), device)
        self.k_scale = None if w.k_scale is None else to_dev(w.k_scale, device)
        self.v_scale = None if w.v_scale is None else to_dev(w.v_scale, device)
        self.torch = torch


def quantize_tokens(x_bits: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """Oracle e4m3 codes of bf16 tokens [T, Hkv, d] with one scale per kv head."""
    import oracle
    x = (x_bits.astype(np.uint32) << 16).view(np.float32)
    out = np.zeros(x.shape, np.uint8)
    for h in range(x.shape[1]):
        out[:, h, :] = oracle.quantize_e4m3(np.ascontiguousarray(x[:, h, :]), float(scale[h]))
    return out


def host_step(w):
    """Oracle side of one step: fork (copy), append (write); returns the
    post-step host caches."""
    import oracle
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    if w.copy_pairs.shape[0]:
        assert oracle.copy_blocks(kc, vc, w.copy_pairs) == 0
    if w.slot_mapping.shape[0]:
        k, v = w.k_new, w.v_new
        if w.dtype == "fp8":
            k, v = quantize_tokens(k, w.k_scale), quantize_tokens(v, w.v_scale)
        assert oracle.kv_cache_write(k, v, w.slot_mapping, kc, vc) == 0
    return kc, vc
