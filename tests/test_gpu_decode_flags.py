"""The opt-in decode flags: PKV_DECODE_ZEROED_WORKSPACE (the split counters are
left at zero by every call, so the zeroing memset can be skipped) and
PKV_DECODE_EARLY_START (programmatic dependent launch behind the append that
writes this step's tokens): results equal the default path bit for bit and the
oracle within tolerance, also inside a CUDA graph."""
import numpy as np
import pytest
import torch

import paged_kv_cache_367_b200 as pkv
from paged_kv_cache_367_b200 import workloads as W
from parity import (assert_close, device_tables, host_pools, oracle_append, oracle_decode,
                    scales, to_f64)

pytestmark = pytest.mark.gpu

C = W.CONFIGS
CFG = {
    "gqa70b": C["gqa70b"].replace(num_seqs=24, lens=("lognormal", 700, 0.9, 16, 4000)),
    "long_splitk": C["long_splitk"].replace(num_seqs=2, lens=("uniform", 4096, 9000)),
    "fp8_prefix": C["fp8_prefix"].replace(num_seqs=12),
}
ZERO, EARLY = pkv.PKV_DECODE_ZEROED_WORKSPACE, pkv.PKV_DECODE_EARLY_START


def _setup(cfg, dev):
    wl = W.make_workload(cfg, device=dev, poison=True)
    bt, lens, slots = device_tables(wl, dev)
    ks, vs = scales(wl, dev)
    c = wl.cfg
    nbytes = pkv.paged_attention_workspace_size(c.num_seqs, c.num_heads, c.num_kv_heads,
                                                c.head_dim, wl.max_seq_len, c.partition_size)
    ws = torch.full((max(nbytes, 1),), 0xAB, dtype=torch.uint8, device=dev)  # garbage
    return wl, bt, lens, slots, ks, vs, ws


def _decode(wl, bt, lens, ks, vs, ws, flags, out=None):
    c = wl.cfg
    out = torch.empty_like(wl.query) if out is None else out
    pkv.paged_attention_decode(out, wl.query, wl.k_cache, wl.v_cache, bt, lens,
                               max_seq_len=wl.max_seq_len, scale=c.scale,
                               partition_size=c.partition_size, workspace=ws, k_scale=ks,
                               v_scale=vs, flags=flags)
    return out


def _counters(ws, c):
    # Workspace layout: partial rows, log-sum-exp values, then the int32 counters.
    g, slots = c.num_heads // c.num_kv_heads, 2 * 1024
    a256 = lambda x: (x + 255) // 256 * 256
    lse = a256(4 * slots * g * c.head_dim)
    done = a256(lse + 4 * slots * g)
    n = c.num_seqs * c.num_kv_heads + 1
    return ws[done:done + 4 * n].view(torch.int32)


@pytest.mark.parametrize("name", list(CFG))
def test_counters_are_left_zero_and_the_memset_can_be_skipped(cuda_dev, name):
    wl, bt, lens, slots, ks, vs, ws = _setup(CFG[name], cuda_dev)
    pkv.paged_kv_append(wl.new_key, wl.new_value, wl.k_cache, wl.v_cache, slots,
                        k_scale=ks, v_scale=vs)
    ref = _decode(wl, bt, lens, ks, vs, ws, 0)
    torch.cuda.synchronize()
    assert torch.all(_counters(ws, wl.cfg) == 0)
    for _ in range(3):
        out = _decode(wl, bt, lens, ks, vs, ws, ZERO)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
        assert torch.all(_counters(ws, wl.cfg) == 0)


@pytest.mark.parametrize("name", list(CFG))
def test_early_start_behind_the_append(cuda_dev, name):
    cfg = CFG[name]
    wl, bt, lens, slots, ks, vs, ws = _setup(cfg, cuda_dev)
    kc, vc = host_pools(wl)
    # Two different new tokens, appended in turn: each decode must see its own.
    gen = torch.Generator(device=cuda_dev).manual_seed(9)
    other_k = torch.randn(wl.new_key.shape, generator=gen, device=cuda_dev).to(wl.new_key.dtype)
    other_v = torch.randn(wl.new_value.shape, generator=gen, device=cuda_dev).to(wl.new_value.dtype)
    pairs = [(wl.new_key, wl.new_value), (other_k, other_v)]
    wants = []
    for nk, nv in pairs:
        wl.new_key, wl.new_value = nk, nv
        k2, v2 = kc.copy(), vc.copy()
        oracle_append(wl, k2, v2)
        wants.append(oracle_decode(wl, k2, v2))
    _decode(wl, bt, lens, ks, vs, ws, 0)  # counters zeroed once
    for it in range(6):
        nk, nv = pairs[it % 2]
        pkv.paged_kv_append(nk, nv, wl.k_cache, wl.v_cache, slots, k_scale=ks, v_scale=vs)
        out = _decode(wl, bt, lens, ks, vs, ws, ZERO | EARLY)
        torch.cuda.synchronize()
        assert pkv.pkv_device_status() == 0
        assert_close(to_f64(out), wants[it % 2], wl.cfg)


def test_early_start_in_a_cuda_graph(cuda_dev):
    wl, bt, lens, slots, ks, vs, ws = _setup(CFG["gqa70b"], cuda_dev)
    kc, vc = host_pools(wl)
    oracle_append(wl, kc, vc)
    want = oracle_decode(wl, kc, vc)
    out = torch.empty_like(wl.query)
    _decode(wl, bt, lens, ks, vs, ws, 0, out)
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        pkv.paged_kv_append(wl.new_key, wl.new_value, wl.k_cache, wl.v_cache, slots)
        _decode(wl, bt, lens, ks, vs, ws, ZERO | EARLY, out)
    for _ in range(5):
        out.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert_close(to_f64(out), want, wl.cfg)
    del graph
