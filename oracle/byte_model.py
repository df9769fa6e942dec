"""KV-cache byte and waste accounting -- test infrastructure.

Plain restatements of the sizing facts the pages give; used to pin the golden
figures printed on the pages and, in the tests, to check the native block
allocator's accounting and the roofline byte counts.

* :func:`kv_cache_size_bytes` -- "KV Cache Optimization and PagedAttention",
  intro: the cache holds K and V, so its size is
  2 x layers x kv heads x head_dim x tokens x batch x bytes per value.
* :func:`unused_slots_contiguous` / :func:`unused_slots_paged` -- the same
  page's worked example of reserving a maximum-length region per request
  versus whole fixed-size blocks: a contiguous reservation wastes
  ``reserved - used`` slots, a paged one only the unused tail of its last
  block (fewer than one block).
"""
from __future__ import annotations


def kv_cache_size_bytes(num_layers: int, num_kv_heads: int, head_dim: int,
                        tokens_per_request: int, num_requests: int,
                        bytes_per_value: int = 2) -> int:
    """Total K+V bytes of a cache holding ``num_requests`` requests of
    ``tokens_per_request`` tokens each."""
    per_token_per_layer = num_kv_heads * head_dim * bytes_per_value
    per_layer = per_token_per_layer * tokens_per_request * num_requests
    return 2 * num_layers * per_layer


def unused_slots_contiguous(tokens_used: int, tokens_reserved: int) -> int:
    """Slots reserved but never written when a request of ``tokens_used`` tokens
    holds a contiguous region sized for ``tokens_reserved``."""
    if tokens_used > tokens_reserved:
        raise ValueError("request longer than its reservation")
    return tokens_reserved - tokens_used


def unused_slots_paged(tokens_used: int, block_size: int) -> int:
    """Slots left empty in the last, partially filled block when a request of
    ``tokens_used`` tokens holds whole blocks of ``block_size`` slots."""
    blocks = -(-tokens_used // block_size)  # ceiling division
    return blocks * block_size - tokens_used


def decode_algorithmic_bytes(seq_lens, num_q_heads: int, num_kv_heads: int,
                             head_dim: int, kv_elem_bytes: int, q_elem_bytes: int,
                             out_elem_bytes: int) -> int:
    """Bytes a decode step must move at minimum: each token's K and V once per
    kv head (the query heads of a group share them), plus q and out."""
    total_tokens = int(sum(int(x) for x in seq_lens))
    kv = 2 * total_tokens * num_kv_heads * head_dim * kv_elem_bytes
    qo = len(seq_lens) * num_q_heads * head_dim * (q_elem_bytes + out_elem_bytes)
    return kv + qo
