"""KV pool fragmentation of a batch of sequence lengths under block policies.

"vLLM 0.5 深度拆解" (chenxutan.com/d/4924) §1.2-§1.3 and "vLLM 推理引擎源码级拆解"
(chenxutan.com/d/5333) §2.1 and §7 describe three ways to hold a batch's K/V:

  * contiguous reservation: every request reserves room for the longest length
    it may reach; the unused tail of the reservation is wasted;
  * fixed-size blocks: a request holds ceil(L / bs) blocks and wastes only the
    free slots of its last block;
  * dynamic page size (p1 §1.3): a request's page size follows its estimated
    length (8 tokens below 128, 16 below 2048, else 32), requests are placed
    longest first, and the small pages of short requests fill the room the
    large pages leave.

Fragmentation is (allocated slots - used slots) / allocated slots. For the
dynamic policy, the plain reading of "placed longest first, small pages fill
the gaps" taken here is first-fit-decreasing packing of the pages into frames
of the largest page size (32 tokens). Page sizes are powers of two that divide
the frame, so packing in decreasing page size leaves no gap except in the last
frame, and the allocated slots are the frames used.
"""
from __future__ import annotations

import numpy as np

DYNAMIC_THRESHOLDS = (128, 2048)
DYNAMIC_PAGE_SIZES = (8, 16, 32)


def fixed_block_fragmentation(lengths, block_size: int) -> float:
    """Unused slots of the last blocks over all allocated slots."""
    L = np.asarray(lengths, dtype=np.int64)
    alloc = int((-(-L // block_size) * block_size).sum())
    return 0.0 if alloc == 0 else (alloc - int(L.sum())) / alloc


def reservation_fragmentation(lengths, max_len: int) -> float:
    """Every request reserves max_len slots; fragmentation of the reservations."""
    L = np.asarray(lengths, dtype=np.int64)
    alloc = max_len * len(L)
    return 0.0 if alloc == 0 else (alloc - int(np.minimum(L, max_len).sum())) / alloc


def dynamic_page_size(estimated_length: int) -> int:
    """Page size for a request of the given estimated length (p1 §1.3)."""
    if estimated_length < DYNAMIC_THRESHOLDS[0]:
        return DYNAMIC_PAGE_SIZES[0]
    if estimated_length < DYNAMIC_THRESHOLDS[1]:
        return DYNAMIC_PAGE_SIZES[1]
    return DYNAMIC_PAGE_SIZES[2]


def dynamic_fragmentation(lengths, estimated=None) -> float:
    """Dynamic page sizes (chosen from `estimated`, default the true lengths),
    pages packed first-fit-decreasing into frames of the largest page size."""
    L = np.asarray(lengths, dtype=np.int64)
    E = L if estimated is None else np.asarray(estimated, dtype=np.int64)
    frame = DYNAMIC_PAGE_SIZES[-1]
    page_slots = 0
    for li, ei in zip(L.tolist(), E.tolist()):
        ps = dynamic_page_size(ei)
        page_slots += -(-li // ps) * ps
    alloc = -(-page_slots // frame) * frame
    return 0.0 if alloc == 0 else (alloc - int(L.sum())) / alloc
