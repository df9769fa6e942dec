"""Brute-force textbook attention on CONTIGUOUS inputs -- test infrastructure.

Used only to pin the oracle (``tests/test_oracle.py``): these functions know
nothing about blocks, block tables or layouts; they take one query row and a
plain [L, d] K and V, straight from the formula Softmax(q K^T / sqrt(d_k)) of
"PagedAttention: Optimizing KV Cache Utilization in Large Language Models",
section "The Math: Block Attention Calculation" (read as one softmax over the
whole sequence), followed by the weighted sum of V rows.
"""
from __future__ import annotations

import math

import numpy as np


def attention_numpy(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * K q) @ V in float64 with numpy's matmul (q [d], K/V [L, d])."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    if K.shape[0] == 0:
        return np.zeros(V.shape[1], dtype=np.float64)
    s = scale * (K @ q)
    w = np.exp(s - s.max())
    w = w / w.sum()
    return w @ V


def attention_loops(q, K, V, scale: float) -> list[float]:
    """The same in pure-Python loops with math.fsum (tiny inputs only)."""
    L = len(K)
    d = len(q)
    if L == 0:
        return [0.0] * d
    s = [scale * math.fsum(float(q[k]) * float(K[t][k]) for k in range(d)) for t in range(L)]
    m = max(s)
    e = [math.exp(x - m) for x in s]
    z = math.fsum(e)
    return [math.fsum(e[t] * float(V[t][k]) for t in range(L)) / z for k in range(d)]


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact upcast of bf16 bit patterns (uint16) to float64."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)
