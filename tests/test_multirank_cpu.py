"""Host logic of the multi-GPU benchmark on CPU: two gloo ranks, as torchrun
would start them. Each rank runs its own replica (distinct seeds, no data-path
collective); timings are reduced by maximum over ranks."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from paged_kv_cache_367_b200 import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        vals = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 3.5], "cpu")
        cfg = W.CONFIGS["gqa70b"].replace(num_seqs=8, seed=bench.replica_seed(1003, rank))
        wl = W.make_workload(cfg, device="cpu")
        lens = bench.max_over_ranks([float(x) for x in wl.seq_lens[:4]], "cpu")
        out[rank] = (vals, list(map(int, wl.seq_lens[:4])), lens)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_by_max_and_use_distinct_replicas():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    (v0, l0, m0), (v1, l1, m1) = out[0], out[1]
    assert v0 == v1 == [2.0, 10.0, 3.5]
    assert l0 != l1                                   # replicas differ
    assert m0 == m1 == [float(max(a, b)) for a, b in zip(l0, l1)]
