"""Fragmentation of block policies (paged_kv_cache_367_b200/fragmentation.py)
against the slot-by-slot simulation in oracle/fragmentation.py, with closed-form
pins from the pages' examples."""
import numpy as np
import pytest

from oracle import fragmentation as O
from paged_kv_cache_367_b200 import fragmentation as F


def test_pins_from_the_pages():
    # "vLLM 推理引擎源码级拆解" §2.2 figure: 7 tokens in blocks of 4 -> 1 free slot of 8.
    assert O.fraction(O.fixed_blocks([7], 4)) == 1 / 8 == F.fixed_block_fragmentation([7], 4)
    # "vLLM 0.5 深度拆解" §1.3: a short request that ends after 10 tokens of a 16-token block.
    assert O.fraction(O.fixed_blocks([10], 16)) == 6 / 16 == F.fixed_block_fragmentation([10], 16)
    # Lengths that fill their blocks waste nothing.
    assert F.fixed_block_fragmentation([16, 32, 48], 16) == 0.0
    # Reservation to the longest length: 1 - mean(L) / max_len.
    assert F.reservation_fragmentation([512, 1024, 2048, 4096], 4096) == pytest.approx(
        1 - 7680 / (4 * 4096))
    # Dynamic page sizes at the thresholds.
    assert [F.dynamic_page_size(x) for x in (1, 127, 128, 2047, 2048, 10**6)] == \
        [8, 8, 16, 16, 32, 32]
    # One 100-token request: 13 pages of 8 = 104 slots, in 4 frames of 32.
    assert O.dynamic_pages([100]) == (128, 100)
    assert F.dynamic_fragmentation([100]) == 28 / 128


@pytest.mark.parametrize("seed", range(5))
def test_closed_forms_equal_the_simulation(seed):
    rng = np.random.default_rng(seed)
    lens = np.concatenate([rng.integers(1, 128, 40), rng.integers(128, 2048, 30),
                           rng.integers(2048, 9000, 5)])
    rng.shuffle(lens)
    for bs in (4, 8, 16, 32):
        assert F.fixed_block_fragmentation(lens, bs) == pytest.approx(
            O.fraction(O.fixed_blocks(lens, bs)), abs=0)
    assert F.reservation_fragmentation(lens, 9000) == pytest.approx(
        O.fraction(O.reservation(lens, 9000)), abs=0)
    est = np.maximum(1, lens + rng.integers(-200, 200, len(lens)))
    for e in (None, est):
        assert F.dynamic_fragmentation(lens, e) == pytest.approx(
            O.fraction(O.dynamic_pages(lens, e)), abs=0)


def test_dynamic_pages_never_waste_more_than_fixed_16_on_short_mixes():
    rng = np.random.default_rng(9)
    lens = rng.integers(16, 160, 128)
    assert F.dynamic_fragmentation(lens) < F.fixed_block_fragmentation(lens, 16)
