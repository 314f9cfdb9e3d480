"""The health word read by pkv_device_status, exercised without a GPU fault.

An expired bounded wait is produced on purpose by the library's self-test
kernel (a wait on a barrier nothing completes, limited to about a millisecond),
and an out-of-pool block id by a decode over a corrupt table. Neither report
may erase the other, and the context stays usable afterwards."""
import pytest
import torch

import paged_kv_cache_367_b200 as pkv
from paged_kv_cache_367_b200 import workloads as W
from parity import gpu_step

pytestmark = pytest.mark.gpu


def test_expired_wait_keeps_the_out_of_pool_report(cuda_dev):
    assert pkv.pkv_device_status(clear=True) == 0
    pkv.pkv_selftest_expired_wait(limit_cycles=1 << 21, note_out_of_pool=True)
    assert pkv.pkv_device_status(clear=False) == 3
    # A second expired wait leaves both values set; clearing resets the word.
    pkv.pkv_selftest_expired_wait(limit_cycles=1 << 21, note_out_of_pool=False)
    assert pkv.pkv_device_status(clear=True) == 3
    assert pkv.pkv_device_status(clear=False) == 0


def test_expired_wait_after_a_corrupt_table_read(cuda_dev):
    cfg = W.CONFIGS["gqa70b"].replace(num_seqs=3, lens=("fixed", [50, 33, 70]), seed=11)
    wl = W.make_workload(cfg, device=cuda_dev)
    bt = wl.block_table.copy()
    bt[1, 0] = wl.num_blocks + 5                     # outside the pool: reads as zeros
    pkv.pkv_device_status(clear=True)
    gpu_step(wl, cuda_dev, block_table=bt)
    pkv.pkv_selftest_expired_wait(limit_cycles=1 << 20, note_out_of_pool=False)
    assert pkv.pkv_device_status(clear=True) == 3
    # The context is still usable: a clean decode reports nothing.
    out = gpu_step(wl, cuda_dev, append=False)
    assert torch.isfinite(out.float()).all()
    assert pkv.pkv_device_status(clear=True) == 0
