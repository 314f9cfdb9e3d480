"""Slot-by-slot simulation of KV pool fragmentation (TEST INFRASTRUCTURE).

Only the test suite may use this module. It allocates explicitly, one token or
one page at a time, the three layouts of "vLLM 0.5 深度拆解" (chenxutan.com/d/4924)
§1.2-§1.3 and "vLLM 推理引擎源码级拆解" (chenxutan.com/d/5333) §2.1-§2.2, and
counts the slots that end up allocated but unused:

  * reservation: each request takes max_len slots up front;
  * fixed blocks: each token fills the next slot of the request's last block,
    or takes a new block when that one is full (p4 §2.2);
  * dynamic page size: page size 8 / 16 / 32 for estimated lengths below 128 /
    below 2048 / longer (p1 §1.3); requests are placed longest first, and each
    page goes to the first 32-slot frame that has a free run of its size at a
    multiple of its size (first fit), else to a new frame.
"""
from __future__ import annotations


def reservation(lengths, max_len):
    alloc = used = 0
    for L in lengths:
        alloc += max_len
        used += min(int(L), max_len)
    return alloc, used


def fixed_blocks(lengths, block_size):
    alloc = used = 0
    for L in lengths:
        blocks, fill = 0, block_size          # fill of the last block (full: none yet)
        for _ in range(int(L)):
            if fill == block_size:
                blocks += 1
                fill = 0
            fill += 1
        alloc += blocks * block_size
        used += int(L)
    return alloc, used


def page_size_for(estimated):
    return 8 if estimated < 128 else (16 if estimated < 2048 else 32)


def dynamic_pages(lengths, estimated=None):
    est = list(lengths) if estimated is None else list(estimated)
    order = sorted(range(len(lengths)), key=lambda i: est[i], reverse=True)
    frames = []                               # each a list of 32 booleans (slot taken)
    used = 0
    for i in order:
        L, ps = int(lengths[i]), page_size_for(est[i])
        used += L
        for _ in range(-(-L // ps)):
            placed = False
            for fr in frames:
                for start in range(0, 32, ps):
                    if not any(fr[start:start + ps]):
                        fr[start:start + ps] = [True] * ps
                        placed = True
                        break
                if placed:
                    break
            if not placed:
                fr = [False] * 32
                fr[:ps] = [True] * ps
                frames.append(fr)
    return 32 * len(frames), used


def fraction(alloc_used):
    alloc, used = alloc_used
    return 0.0 if alloc == 0 else (alloc - used) / alloc
