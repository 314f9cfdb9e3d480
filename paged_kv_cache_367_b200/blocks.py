"""Host block manager (C ABI in include/pagedkv_blocks.h): the ledger that hands
out slots, block tables and copy lists for the kernels. A ctypes wrapper only;
the bookkeeping runs in the library's native code."""
from __future__ import annotations

import ctypes

import numpy as np

from . import PagedKVError, load_library

_I64P = ctypes.POINTER(ctypes.c_int64)


def _check(fn: str, st: int) -> None:
    if st != 0:
        raise PagedKVError(fn, st)


class BlockManager:
    """num_blocks device blocks and num_host_blocks host (swap) blocks of
    block_size tokens; prefix_caching names full blocks by their hash chain."""

    def __init__(self, num_blocks: int, block_size: int, num_host_blocks: int = 0,
                 prefix_caching: bool = False):
        self._lib = load_library()
        self.block_size = block_size
        self.num_blocks = num_blocks
        self.num_host_blocks = num_host_blocks
        self._h = self._lib.pkv_bm_create(num_blocks, num_host_blocks, block_size,
                                          1 if prefix_caching else 0)
        if not self._h:
            raise ValueError("pkv_bm_create failed (bad sizes or out of memory)")

    def close(self) -> None:
        if getattr(self, "_h", None):
            self._lib.pkv_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    @property
    def num_free(self) -> int:
        return self._lib.pkv_bm_num_free(self._h)

    @property
    def num_free_host(self) -> int:
        return self._lib.pkv_bm_num_free_host(self._h)

    def can_allocate(self, num_tokens: int) -> bool:
        return bool(self._lib.pkv_bm_can_allocate(self._h, num_tokens))

    def allocate(self, seq_id: int, token_ids) -> tuple[np.ndarray, int]:
        """Admit a prompt; returns (slot_mapping int64 [n], -1 for cached tokens;
        number of leading cached tokens)."""
        tok = np.ascontiguousarray(token_ids, dtype=np.int32)
        slots = np.empty(len(tok), dtype=np.int64)
        cached = ctypes.c_int64(0)
        _check("pkv_bm_allocate", self._lib.pkv_bm_allocate(
            self._h, seq_id, tok.ctypes.data if len(tok) else None, len(tok),
            slots.ctypes.data if len(tok) else None, ctypes.byref(cached)))
        return slots, cached.value

    def can_append(self, seq_id: int) -> bool:
        return bool(self._lib.pkv_bm_can_append(self._h, seq_id))

    def append_slot(self, seq_id: int, token_id: int = 0) -> tuple[int, int, int]:
        """Slot of the sequence's next token and the copy-on-write pair
        (src, dst), or (-1, -1)."""
        slot, src, dst = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        _check("pkv_bm_append_slot", self._lib.pkv_bm_append_slot(
            self._h, seq_id, int(token_id), ctypes.byref(slot), ctypes.byref(src),
            ctypes.byref(dst)))
        return slot.value, src.value, dst.value

    def append_slots(self, seq_ids, token_ids) -> tuple[np.ndarray, np.ndarray]:
        """One decode step for a batch: (slot_mapping int64 [n], copy-on-write
        pairs int64 [m, 2] to copy before the append). All or nothing."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        tok = np.ascontiguousarray(token_ids, dtype=np.int32)
        if len(tok) != len(ids):
            raise ValueError("seq_ids and token_ids differ in length")
        slots = np.empty(len(ids), dtype=np.int64)
        cow = np.empty((max(len(ids), 1), 2), dtype=np.int64)
        m = ctypes.c_int64(0)
        _check("pkv_bm_append_slots", self._lib.pkv_bm_append_slots(
            self._h, ids.ctypes.data, tok.ctypes.data, len(ids), slots.ctypes.data,
            cow.ctypes.data, ctypes.byref(m)))
        return slots, cow[:m.value].copy()

    def fork(self, parent_id: int, child_id: int) -> None:
        _check("pkv_bm_fork", self._lib.pkv_bm_fork(self._h, parent_id, child_id))

    def free(self, seq_id: int) -> None:
        _check("pkv_bm_free", self._lib.pkv_bm_free(self._h, seq_id))

    def _swap(self, fn: str, seq_ids) -> np.ndarray:
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        cap = self.num_blocks + self.num_host_blocks
        pairs = np.empty((max(cap, 1), 2), dtype=np.int64)
        n = ctypes.c_int64(0)
        _check(fn, getattr(self._lib, fn)(self._h, ids.ctypes.data if len(ids) else None,
                                          len(ids), pairs.ctypes.data, cap, ctypes.byref(n)))
        return pairs[:n.value].copy()

    def swap_out(self, seq_ids) -> np.ndarray:
        """(device block, host block) pairs to copy out, [n, 2] int64."""
        return self._swap("pkv_bm_swap_out", seq_ids)

    def swap_in(self, seq_ids) -> np.ndarray:
        """(host block, device block) pairs to copy in, [n, 2] int64."""
        return self._swap("pkv_bm_swap_in", seq_ids)

    def block_tables(self, seq_ids, max_blocks_per_seq: int) -> tuple[np.ndarray, np.ndarray]:
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        table = np.empty((len(ids), max_blocks_per_seq), dtype=np.int32)
        lens = np.empty(len(ids), dtype=np.int32)
        _check("pkv_bm_block_tables", self._lib.pkv_bm_block_tables(
            self._h, ids.ctypes.data if len(ids) else None, len(ids), max_blocks_per_seq,
            table.ctypes.data if len(ids) else None, lens.ctypes.data if len(ids) else None))
        return table, lens

    def seq_len(self, seq_id: int) -> int:
        n = self._lib.pkv_bm_seq_len(self._h, seq_id)
        if n < 0:
            raise PagedKVError("pkv_bm_seq_len", n)
        return n

    def refcount(self, block: int) -> int:
        return self._lib.pkv_bm_refcount(self._h, block)

    def usage(self) -> dict:
        """Pool usage: blocks held / cached-unheld / free, resident tokens, used
        slots of held blocks, and the held blocks' fragmentation."""
        out = np.zeros(6, dtype=np.int64)
        _check("pkv_bm_usage", self._lib.pkv_bm_usage(self._h, out.ctypes.data))
        nb, held, cached, free, tokens, used = (int(x) for x in out)
        return {"num_blocks": nb, "held": held, "cached_unheld": cached, "free": free,
                "usage": held / nb if nb else 0.0, "tokens": tokens, "used_slots": used,
                "fragmentation": 1.0 - used / (held * self.block_size) if held else 0.0}

    def check(self) -> None:
        _check("pkv_bm_check", self._lib.pkv_bm_check(self._h))
