"""paged_attention_decode_static: the decode entry point for callers that cannot
allocate device memory (its split scratch is a fixed array inside the library).
Called through the C ABI, it must give the same output as paged_attention_decode
with a caller workspace, within the decode tolerance, on two calls in a row (the
second call finds the array holding the first call's contents). This file is
collected last so that a run stopping at the first failure has already run
every other test."""
import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_367_b200 as pkv
from paged_kv_cache_367_b200 import workloads as W
from parity import TOL, device_tables

pytestmark = pytest.mark.gpu


def _static_call(lib, out, wl, bt, lens, P):
    c = wl.cfg
    S, Hq, D = wl.query.shape
    nb, bs, Hkv, _ = wl.k_cache.shape
    return lib.paged_attention_decode_static(
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(wl.query.data_ptr()),
        ctypes.c_void_p(wl.k_cache.data_ptr()), ctypes.c_void_p(wl.v_cache.data_ptr()),
        ctypes.c_void_p(bt.data_ptr()), ctypes.c_void_p(lens.data_ptr()), S, Hq, Hkv, D, bs,
        wl.block_table.shape[1], nb, wl.max_seq_len, ctypes.c_float(c.scale), pkv.PKV_BF16,
        pkv.PKV_BF16, None, None, P, 0, 0, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_static_scratch_decode_matches_workspace_decode_twice(cuda_dev):
    lib = pkv.load_library()
    cfg = W.CONFIGS["gqa70b"].replace(num_seqs=24, lens=("lognormal", 700, 0.8, 16, 3000),
                                      seed=2024)
    wl = W.make_workload(cfg, device=cuda_dev)
    bt, lens, _ = device_tables(wl, cuda_dev)
    P = 64                                           # many split sequences
    ref = torch.empty_like(wl.query)
    nbytes = pkv.paged_attention_workspace_size(cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads,
                                                cfg.head_dim, wl.max_seq_len, P)
    assert nbytes > 0
    ws = torch.empty(nbytes, dtype=torch.uint8, device=cuda_dev)
    pkv.paged_attention_decode(ref, wl.query, wl.k_cache, wl.v_cache, bt, lens,
                               max_seq_len=wl.max_seq_len, scale=cfg.scale, partition_size=P,
                               workspace=ws)
    tmax, tmean = TOL["bf16"]
    want = ref.float().cpu().numpy()
    for _ in range(2):
        out = torch.full_like(wl.query, float("nan"))
        assert _static_call(lib, out, wl, bt, lens, P) == 0
        torch.cuda.synchronize()
        got = out.float().cpu().numpy()
        assert np.all(np.isfinite(got))
        err = np.abs(got - want)
        assert err.max() <= tmax and err.mean() <= tmean
    assert pkv.pkv_device_status(clear=True) == 0


def test_static_scratch_rejects_sizes_beyond_its_limit(cuda_dev):
    lib = pkv.load_library()
    cfg = W.CONFIGS["gqa70b"].replace(num_seqs=2, num_heads=32, num_kv_heads=2,
                                      lens=("fixed", [600, 300]), seed=7)
    wl = W.make_workload(cfg, device=cuda_dev)
    bt, lens, _ = device_tables(wl, cuda_dev)
    out = torch.empty_like(wl.query)
    # 16 query heads per KV head at head_dim 128 need more than the fixed 16 MiB.
    assert pkv.paged_attention_workspace_size(2, 32, 2, 128, wl.max_seq_len, 64) > 16 << 20
    assert _static_call(lib, out, wl, bt, lens, 64) == -5       # PKV_ERR_WORKSPACE
