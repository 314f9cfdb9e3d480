"""paged_attention_decode_static: the decode entry point for callers that cannot
allocate device memory (its split scratch is a fixed array inside the library).
Called through the C ABI, it must give the same output as paged_attention_decode
with a caller workspace, and the fp64 oracle's within the decode tolerance, on
two calls in a row (the second call finds the array holding the first call's
contents), and also when consecutive calls change the group size and head_dim
(which moves the counters inside the shared array) or pass
PKV_DECODE_ZEROED_WORKSPACE (which this entry point must ignore). This file is
collected last so that a run stopping at the first failure has already run
every other test."""
import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_367_b200 as pkv
from paged_kv_cache_367_b200 import workloads as W
from parity import TOL, assert_close, device_tables, host_pools, oracle_append, oracle_decode

pytestmark = pytest.mark.gpu


def _static_call(lib, out, wl, bt, lens, P, flags=0):
    c = wl.cfg
    S, Hq, D = wl.query.shape
    nb, bs, Hkv, _ = wl.k_cache.shape
    return lib.paged_attention_decode_static(
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(wl.query.data_ptr()),
        ctypes.c_void_p(wl.k_cache.data_ptr()), ctypes.c_void_p(wl.v_cache.data_ptr()),
        ctypes.c_void_p(bt.data_ptr()), ctypes.c_void_p(lens.data_ptr()), S, Hq, Hkv, D, bs,
        wl.block_table.shape[1], nb, wl.max_seq_len, ctypes.c_float(c.scale), pkv.PKV_BF16,
        pkv.PKV_BF16, None, None, P, 0, flags,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _workspace_decode(wl, bt, lens, P, dev):
    c = wl.cfg
    ref = torch.empty_like(wl.query)
    nbytes = pkv.paged_attention_workspace_size(c.num_seqs, c.num_heads, c.num_kv_heads,
                                                c.head_dim, wl.max_seq_len, P)
    assert nbytes > 0
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    pkv.paged_attention_decode(ref, wl.query, wl.k_cache, wl.v_cache, bt, lens,
                               max_seq_len=wl.max_seq_len, scale=c.scale, partition_size=P,
                               workspace=ws)
    torch.cuda.synchronize()
    return ref.float().cpu().numpy()


def _case(dev, seed, num_heads, head_dim, num_seqs=24):
    """A poisoned workload with this step's tokens appended on the GPU, and the
    oracle's output for it."""
    cfg = W.CONFIGS["gqa70b"].replace(num_seqs=num_seqs, num_heads=num_heads, head_dim=head_dim,
                                      lens=("lognormal", 700, 0.8, 16, 3000), seed=seed)
    wl = W.make_workload(cfg, device=dev, poison=True)
    bt, lens, slots = device_tables(wl, dev)
    kc, vc = host_pools(wl)
    oracle_append(wl, kc, vc)
    pkv.paged_kv_append(wl.new_key, wl.new_value, wl.k_cache, wl.v_cache, slots)
    return wl, bt, lens, oracle_decode(wl, kc, vc)


def _check_static(lib, wl, bt, lens, P, want_ws, want_oracle, flags=0):
    out = torch.full_like(wl.query, float("nan"))
    assert _static_call(lib, out, wl, bt, lens, P, flags) == 0
    torch.cuda.synchronize()
    got = out.float().cpu().numpy()
    assert np.all(np.isfinite(got))
    tmax, tmean = TOL["bf16"]
    err = np.abs(got - want_ws)
    assert err.max() <= tmax and err.mean() <= tmean, "static vs workspace decode"
    assert_close(got.astype(np.float64), want_oracle, wl.cfg, "static vs oracle")


def test_static_scratch_decode_matches_workspace_decode_twice(cuda_dev):
    lib = pkv.load_library()
    wl, bt, lens, want_oracle = _case(cuda_dev, 2024, 64, 128)
    P = 64                                           # many split sequences
    want_ws = _workspace_decode(wl, bt, lens, P, cuda_dev)
    for _ in range(2):
        _check_static(lib, wl, bt, lens, P, want_ws, want_oracle)
    assert pkv.pkv_device_status(clear=True) == 0


def test_static_scratch_survives_shape_changes_and_ignores_zeroed_flag(cuda_dev):
    # g = 8, head_dim 128; then g = 4, head_dim 64 (its counters sit where the
    # first call left partial rows) with PKV_DECODE_ZEROED_WORKSPACE; then the
    # first shape again with the flag.
    lib = pkv.load_library()
    P = 64
    cases = []
    for seed, Hq, D in ((31, 64, 128), (32, 32, 64)):
        wl, bt, lens, want_oracle = _case(cuda_dev, seed, Hq, D)
        cases.append((wl, bt, lens, _workspace_decode(wl, bt, lens, P, cuda_dev), want_oracle))
    flag = pkv.PKV_DECODE_ZEROED_WORKSPACE
    for k, f in ((0, 0), (1, flag), (0, flag), (1, 0)):
        wl, bt, lens, want_ws, want_oracle = cases[k]
        _check_static(lib, wl, bt, lens, P, want_ws, want_oracle, flags=f)
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
