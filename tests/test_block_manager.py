"""Host block manager (include/pagedkv_blocks.h) against the plain logical model
(oracle/block_model.py): worked cases from the pages, error behaviour, and
random traces whose pool contents are simulated on the CPU with the oracle's
plain block copy. Needs no GPU."""
import numpy as np
import pytest

from blocktrace import NumpyPools, Trace
from oracle import block_model as M
from paged_kv_cache_367_b200 import PagedKVError
from paged_kv_cache_367_b200.blocks import BlockManager

ENO_BLOCKS, ESEQ, ESHAPE = -8, -9, -2


def status(exc):
    return exc.value.status


def test_figure_request_fills_last_block_then_takes_a_new_one():
    # "vLLM 推理引擎源码级拆解" §2.2: bs 4, a 7-token request holds 2 blocks; the
    # 8th token fills the last block's free slot, the 9th takes a new block.
    bm = BlockManager(8, 4)
    slots, cached = bm.allocate(1, list(range(7)))
    assert cached == 0 and bm.num_free == 6
    table, lens = bm.block_tables([1], 4)
    b0, b1 = table[0, :2]
    assert list(slots) == [b0 * 4 + t for t in range(4)] + [b1 * 4 + t for t in range(3)]
    slot, src, dst = bm.append_slot(1, 7)
    assert (slot, src, dst) == (b1 * 4 + 3, -1, -1) and bm.num_free == 6
    slot, src, dst = bm.append_slot(1, 8)
    table, lens = bm.block_tables([1], 4)
    assert table[0, 2] >= 0 and slot == table[0, 2] * 4 and lens[0] == 9 and bm.num_free == 5
    bm.check()


def test_blocks_per_sequence_worked_examples():
    # "vLLM 深度实战" §1.2: 48 tokens hold 3 blocks of 16, 200 tokens hold 13.
    bm = BlockManager(16, 16)
    bm.allocate(1, [0] * 48)
    bm.allocate(2, [])                          # admitted empty, grows below
    for _ in range(200):
        bm.append_slot(2, 0)
    table, lens = bm.block_tables([1, 2], 13)
    assert list(lens) == [48, 200]
    assert (table[0] >= 0).sum() == 3 and (table[1] >= 0).sum() == 13
    assert bm.num_free == 0
    bm.free(1)
    bm.free(2)
    assert bm.num_free == 16
    bm.check()


def test_fork_then_copy_on_write_of_the_shared_partial_block():
    bm = BlockManager(8, 4)
    bm.allocate(1, [1, 2, 3, 4, 5, 6])   # blocks: full, partial (2 tokens)
    bm.fork(1, 2)
    t1, _ = bm.block_tables([1], 2)
    shared_last = int(t1[0, 1])
    assert bm.refcount(int(t1[0, 0])) == 2 and bm.refcount(shared_last) == 2
    slot, src, dst = bm.append_slot(2, 7)      # child writes first: copy
    assert src == shared_last and dst >= 0 and dst != src and slot == dst * 4 + 2
    assert bm.refcount(shared_last) == 1 and bm.refcount(dst) == 1
    slot, src, dst = bm.append_slot(1, 9)      # parent now owns its block alone
    assert (src, dst) == (-1, -1) and slot == shared_last * 4 + 2
    bm.check()


def test_fork_at_a_block_boundary_needs_no_copy():
    bm = BlockManager(8, 4)
    bm.allocate(1, [1, 2, 3, 4])
    bm.fork(1, 2)
    for sid in (1, 2):
        slot, src, dst = bm.append_slot(sid, 5)
        assert (src, dst) == (-1, -1)
    t, _ = bm.block_tables([1, 2], 2)
    assert t[0, 0] == t[1, 0] and t[0, 1] != t[1, 1]
    bm.check()


def test_out_of_blocks_changes_nothing():
    bm = BlockManager(4, 4, prefix_caching=True)
    bm.allocate(1, list(range(10)))            # 3 blocks
    assert not bm.can_allocate(8)
    with pytest.raises(PagedKVError) as e:
        bm.allocate(2, list(range(100, 108)))
    assert status(e) == ENO_BLOCKS
    bm.check()
    assert bm.num_free == 1
    with pytest.raises(PagedKVError) as e:
        bm.seq_len(2)
    assert status(e) == ESEQ
    bm.append_slot(1, 10)
    bm.append_slot(1, 11)                       # fills block 3 (the partial one)
    assert bm.can_append(1)                     # one free block left
    bm.append_slot(1, 12)                       # takes the last free block
    for tok in (13, 14, 15):
        assert bm.can_append(1)
        bm.append_slot(1, tok)
    assert not bm.can_append(1)                 # full, and no block left
    with pytest.raises(PagedKVError) as e:
        bm.append_slot(1, 0)
    assert status(e) == ENO_BLOCKS
    assert bm.seq_len(1) == 16
    bm.check()


def test_error_codes():
    bm = BlockManager(4, 4, num_host_blocks=1)
    bm.allocate(1, [1, 2])
    for call in (lambda: bm.allocate(1, [3]), lambda: bm.fork(9, 2), lambda: bm.fork(1, 1),
                 lambda: bm.free(9), lambda: bm.append_slot(9), lambda: bm.swap_in([1]),
                 lambda: bm.swap_out([1, 1])):
        with pytest.raises(PagedKVError) as e:
            call()
        assert status(e) == ESEQ
    bm.allocate(2, [1] * 9)                     # 3 blocks
    with pytest.raises(PagedKVError) as e:
        bm.block_tables([2], 2)
    assert status(e) == ESHAPE
    with pytest.raises(PagedKVError) as e:
        bm.swap_out([2])                        # 3 blocks, 1 host block
    assert status(e) == ENO_BLOCKS
    bm.swap_out([1])
    with pytest.raises(PagedKVError) as e:
        bm.append_slot(1)
    assert status(e) == ESEQ
    with pytest.raises(PagedKVError) as e:
        bm.block_tables([1], 4)
    assert status(e) == ESEQ
    bm.check()


def test_prefix_cache_shares_whole_matching_blocks_only():
    bs = 4
    bm = BlockManager(32, bs, prefix_caching=True)
    system = [7, 7, 1, 2, 3, 9, 9, 4]           # two full blocks
    s1, c1 = bm.allocate(1, system + [5, 6])
    assert c1 == 0 and np.all(s1 >= 0)
    s2, c2 = bm.allocate(2, system + [5, 6, 8])  # same two blocks, own partial tail
    assert c2 == 8 and np.all(s2[:8] == -1) and np.all(s2[8:] >= 0)
    t, _ = bm.block_tables([1, 2], 3)
    assert list(t[0, :2]) == list(t[1, :2]) and t[0, 2] != t[1, 2]
    # The same 4 tokens after a different first block name a different block.
    s3, c3 = bm.allocate(3, [0, 0, 0, 0] + system[4:])
    t3, _ = bm.block_tables([3], 2)
    assert c3 == 0 and t3[0, 1] != t[0, 1]
    # A request that diverges inside block 0 shares nothing.
    s4, c4 = bm.allocate(4, [7, 7, 1, 0] + system[4:])
    assert c4 == 0
    # Appends that complete a block name it: the next request hits it.
    bm.allocate(5, system + [5, 6])
    for tok in (8, 8):
        bm.append_slot(5, tok)                  # block 2 of seq 5 = [5, 6, 8, 8]
    s6, c6 = bm.allocate(6, system + [5, 6, 8, 8, 1])
    assert c6 == 12
    t56, _ = bm.block_tables([5, 6], 4)
    assert t56[0, 2] == t56[1, 2]
    bm.check()


def test_prefix_cache_blocks_survive_free_and_are_evicted_lru_first():
    bs = 4
    bm = BlockManager(4, bs, prefix_caching=True)
    a, b = [1, 1, 1, 1], [2, 2, 2, 2]
    bm.allocate(1, a)
    bm.allocate(2, b)
    ta, _ = bm.block_tables([1], 1)
    tb, _ = bm.block_tables([2], 1)
    bm.free(1)                                   # a becomes cached-unheld first
    bm.free(2)
    assert bm.num_free == 4
    _, c = bm.allocate(3, a)                     # hit: a is held again
    assert c == 4 and bm.block_tables([3], 1)[0][0, 0] == ta[0, 0]
    bm.free(3)                                   # now b is least recent, then a
    bm.allocate(4, [9] * 12)                     # 3 blocks: 2 free, then evict b
    _, cb = bm.allocate(5, b)                    # b was evicted: a miss
    assert cb == 0
    bm.free(4)
    bm.free(5)
    _, ca = bm.allocate(6, a)                    # a was evicted after b
    bm.check()
    assert ca == 0


def test_swap_out_and_in_keeps_sharing_within_the_group():
    bm = BlockManager(8, 4, num_host_blocks=8)
    bm.allocate(1, list(range(6)))
    bm.fork(1, 2)
    bm.allocate(3, [1, 2])
    pairs = bm.swap_out([1, 2])
    assert len(pairs) == 2                       # two distinct blocks, shared by both
    assert bm.num_free == 7 and bm.num_free_host == 6
    bm.check()
    back = bm.swap_in([2, 1])
    assert sorted(back[:, 0].tolist()) == sorted(pairs[:, 1].tolist())
    t, lens = bm.block_tables([1, 2], 2)
    assert list(t[0]) == list(t[1]) and list(lens) == [6, 6]
    assert bm.num_free_host == 8
    bm.check()


@pytest.mark.parametrize("prefix", [False, True])
@pytest.mark.parametrize("seed", range(6))
def test_random_traces_preserve_every_sequence(prefix, seed):
    bs = (4, 8, 16)[seed % 3]
    pools = NumpyPools(48, 24, bs, (1, 4))
    tr = Trace(pools, num_blocks=48, bs=bs, num_host_blocks=24, prefix_caching=prefix,
               seed=seed)
    for i in range(600):
        tr.step()
        tr.check_ledger()
        if i % 10 == 0:
            tr.check_contents(*pools.device_pools())
    tr.check_contents(*pools.device_pools())
    st = tr.stats
    assert st["cow"] > 0 and st["swap_out"] > 0 and st["swap_in"] > 0
    if prefix:
        assert st["cached"] > 0


def test_batched_step_equals_one_call_per_sequence():
    rng = np.random.default_rng(3)
    a, b = BlockManager(64, 4, prefix_caching=True), BlockManager(64, 4, prefix_caching=True)
    for bm in (a, b):
        bm.allocate(1, [1, 2, 3, 4, 5, 6])
        bm.allocate(2, [1, 2, 3, 4, 5, 6])          # shares the first block
        bm.fork(1, 3)                                # shares both blocks of 1
        bm.allocate(4, [])
    for _ in range(9):
        ids = [3, 1, 4, 2]
        toks = rng.integers(0, 9, size=4)
        slots, cow = a.append_slots(ids, toks)
        want = [b.append_slot(i, int(t)) for i, t in zip(ids, toks)]
        assert list(slots) == [w[0] for w in want]
        assert cow.tolist() == [[w[1], w[2]] for w in want if w[1] >= 0]
    for bm in (a, b):
        bm.check()
    ta, _ = a.block_tables([1, 2, 3, 4], 5)
    tb, _ = b.block_tables([1, 2, 3, 4], 5)
    assert np.array_equal(ta, tb)


def test_batched_step_is_all_or_nothing():
    bm = BlockManager(3, 4)
    bm.allocate(1, [0] * 4)                          # full: the next token needs a block
    bm.allocate(2, [0] * 4)
    bm.allocate(3, [0] * 2)                          # partial: writes in place
    with pytest.raises(PagedKVError) as e:
        bm.append_slots([1, 2, 3], [0, 0, 0])        # 2 blocks needed, 0 free
    assert status(e) == ENO_BLOCKS
    assert [bm.seq_len(i) for i in (1, 2, 3)] == [4, 4, 2]
    slots, cow = bm.append_slots([3], [5])
    assert len(cow) == 0 and bm.seq_len(3) == 3
    for ids in ([3, 3], [9], [1, 9]):
        with pytest.raises(PagedKVError) as e:
            bm.append_slots(ids, [0] * len(ids))
        assert status(e) == ESEQ
    bm.check()


def test_usage_metrics():
    from paged_kv_cache_367_b200 import fragmentation as FR
    bm = BlockManager(32, 4, prefix_caching=True)
    lens = [7, 4, 10]
    for i, L in enumerate(lens):
        bm.allocate(i, list(range(100 * i, 100 * i + L)))  # nothing shared
    u = bm.usage()
    assert (u["num_blocks"], u["held"], u["cached_unheld"], u["free"]) == (32, 6, 0, 26)
    assert u["tokens"] == 21 and u["used_slots"] == 21
    assert u["fragmentation"] == pytest.approx(FR.fixed_block_fragmentation(lens, 4))
    bm.fork(0, 9)                                     # shares seq 0's two blocks
    u = bm.usage()
    assert u["held"] == 6 and u["tokens"] == 28 and u["used_slots"] == 21
    bm.free(1)                                        # its full block stays cached
    u = bm.usage()
    assert (u["held"], u["cached_unheld"], u["free"]) == (5, 1, 26)
    bm.check()


def test_model_blocks_needed_closed_form():
    assert [M.blocks_needed(n, 16) for n in (0, 1, 16, 17, 48, 200)] == [0, 1, 1, 2, 3, 13]
