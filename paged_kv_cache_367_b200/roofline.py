"""Algorithmic byte counts for the roofline of the paged decode path.

The per-token KV size follows the formula in "vLLM 推理引擎源码级拆解"
(chenxutan.com/d/5333) §1: 2 (K and V) x layers x KV heads x head_dim x element
bytes. One decode step of one layer reads, per sequence, exactly its seq_len
tokens of K and V for every KV head, its query rows, its block-table entries
and length, and writes its output rows:

    bytes = 2 * T * Hkv * D * e_kv + S * Hq * D * e_q (query) + S * Hq * D * e_q
            (output) + 4 * sum(ceil(L_i / bs)) (block table) + 4 * S (seq_lens)

with T = sum(L_i). Padded slots of a sequence's last block and the split-K
workspace are overhead the kernel pays, not algorithmic bytes. Where sequences
share prefix blocks, `shared_prefix_tokens` counts those tokens' K/V once
(the bytes HBM must deliver) instead of once per sequence.
"""
from __future__ import annotations

from typing import Iterable


def kv_bytes_per_token(num_layers: int, num_kv_heads: int, head_dim: int, elem_bytes: int) -> int:
    return 2 * num_layers * num_kv_heads * head_dim * elem_bytes


def decode_bytes(seq_lens: Iterable[int], num_heads: int, num_kv_heads: int, head_dim: int,
                 block_size: int, q_bytes: int, kv_bytes: int,
                 shared_prefix_tokens: int = 0) -> int:
    lens = [max(0, int(L)) for L in seq_lens]
    S = len(lens)
    T = sum(lens)
    if shared_prefix_tokens and S:
        T = T - shared_prefix_tokens * (S - 1)
    blocks = sum(-(-L // block_size) for L in lens)
    kv = T * kv_bytes_per_token(1, num_kv_heads, head_dim, kv_bytes)
    qo = 2 * S * num_heads * head_dim * q_bytes
    return kv + qo + 4 * blocks + 4 * S


def append_bytes(num_tokens: int, num_kv_heads: int, head_dim: int, src_bytes: int,
                 cache_bytes: int) -> int:
    """K and V rows read (src) and written (cache), plus the int64 slot of each token."""
    return 2 * num_tokens * num_kv_heads * head_dim * (src_bytes + cache_bytes) + 8 * num_tokens
