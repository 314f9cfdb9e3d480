"""Plain model of what the block manager must preserve (TEST INFRASTRUCTURE).

Only the test suite may use this module. It restates, without any paging, the
observable contract of the KV block ledger in "vLLM 推理引擎源码级拆解"
(chenxutan.com/d/5333) §2.1-§2.2, §3.1-§3.2 and §4.2, and "vLLM 深度实战"
(chenxutan.com/d/3332) §1.2:

  * each live sequence is an ordered list of tokens whose K/V rows it alone
    sees; paging, sharing, copy-on-write, swapping and prefix caching must
    never change those rows (a fork starts with a copy of the parent's list,
    and later appends to either touch only that one);
  * a sequence of L tokens holds ceil(L / block_size) blocks (a finished or
    preempted one holds none), and a block is shared only by sequences whose
    tokens in it, and all tokens before it, are equal;
  * the free count is the pool size minus the distinct blocks held.

It also holds the plain whole-block copy (K and V of src to dst, pair by pair)
that copy-on-write and swapping apply to a pool.
"""
from __future__ import annotations

import numpy as np


class LogicalSequences:
    """Sequences as contiguous token lists with their K/V rows (no paging)."""

    def __init__(self):
        self.tokens: dict[int, list[int]] = {}
        self.k: dict[int, list[np.ndarray]] = {}
        self.v: dict[int, list[np.ndarray]] = {}

    def add(self, seq_id, token_ids, k_rows, v_rows):
        assert seq_id not in self.tokens
        self.tokens[seq_id] = list(token_ids)
        self.k[seq_id] = [np.array(r) for r in k_rows]
        self.v[seq_id] = [np.array(r) for r in v_rows]

    def append(self, seq_id, token_id, k_row, v_row):
        self.tokens[seq_id].append(token_id)
        self.k[seq_id].append(np.array(k_row))
        self.v[seq_id].append(np.array(v_row))

    def fork(self, parent, child):
        assert child not in self.tokens
        self.tokens[child] = list(self.tokens[parent])
        self.k[child] = [r.copy() for r in self.k[parent]]
        self.v[child] = [r.copy() for r in self.v[parent]]

    def remove(self, seq_id):
        del self.tokens[seq_id], self.k[seq_id], self.v[seq_id]

    def length(self, seq_id) -> int:
        return len(self.tokens[seq_id])

    def rows(self, seq_id):
        """(K [L, ...], V [L, ...]) of the sequence, in token order."""
        k, v = self.k[seq_id], self.v[seq_id]
        if not k:
            return None, None
        return np.stack(k), np.stack(v)


def blocks_needed(length: int, block_size: int) -> int:
    """Blocks a sequence of `length` tokens holds: ceil(length / block_size)."""
    return -(-length // block_size)


def copy_blocks(src_k, src_v, dst_k, dst_v, pairs) -> None:
    """For each (src, dst) pair in order: dst pools' block dst = src pools'
    block src (K and V), byte for byte. In-pool copies pass the same arrays."""
    for s, d in np.asarray(pairs, dtype=np.int64).reshape(-1, 2):
        dst_k[d] = src_k[s]
        dst_v[d] = src_v[s]


def gather(pool, table_row, length: int, block_size: int):
    """The `length` token rows a block-table row points at, in token order."""
    out = [pool[table_row[t // block_size], t % block_size] for t in range(length)]
    return np.stack(out) if out else None
