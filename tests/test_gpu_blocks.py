"""Block copies (copy-on-write, swap to pinned host memory) through the C ABI,
byte for byte against the oracle's plain copy, and a block-manager trace run
with the library's kernels (append, copy-on-write copies, swaps) whose pool
and decode outputs are checked against the plain logical model and the fp64
oracle."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_367_b200 as pkv
from blocktrace import Trace
from oracle import block_model as M
from paged_kv_cache_367_b200 import workloads as W
from paged_kv_cache_367_b200.blocks import BlockManager
from parity import TOL

pytestmark = pytest.mark.gpu


def _pool(nb, bs, Hkv, D, dtype, dev, gen):
    if dtype == torch.uint8:
        return torch.randint(0, 256, (nb, bs, Hkv, D), dtype=torch.uint8, generator=gen).to(dev)
    return torch.randn((nb, bs, Hkv, D), generator=gen).to(dtype).to(dev)


def _pairs(nb, n, rng, out_of_range=0):
    ids = rng.permutation(nb)[:2 * n].reshape(n, 2)      # distinct blocks: no overlap
    ids = ids.astype(np.int64)
    if out_of_range:
        ids[:out_of_range, rng.integers(2)] = nb + 5      # copies nothing
        ids[out_of_range:2 * out_of_range, 0] = -1
    return ids


@pytest.mark.parametrize("bs,Hkv,D,dtype", [(16, 8, 128, torch.bfloat16), (8, 1, 64, torch.float16),
                                             (32, 8, 128, torch.uint8), (16, 40, 128, torch.float16)])
@pytest.mark.parametrize("n", [1, 7, 300])
def test_copy_blocks_bit_exact(cuda_dev, bs, Hkv, D, dtype, n):
    gen = torch.Generator().manual_seed(n)
    nb = 2 * n + 40
    k = _pool(nb, bs, Hkv, D, dtype, cuda_dev, gen)
    v = _pool(nb, bs, Hkv, D, dtype, cuda_dev, gen)
    pairs = _pairs(nb, n, np.random.default_rng(n), out_of_range=min(2, n // 3))
    want_k, want_v = W.host(k).copy(), W.host(v).copy()
    ok = (pairs >= 0).all(1) & (pairs < nb).all(1)
    M.copy_blocks(want_k, want_v, want_k, want_v, pairs[ok])
    pkv.paged_kv_copy_blocks(k, v, torch.from_numpy(pairs).to(cuda_dev))
    torch.cuda.synchronize()
    assert np.array_equal(W.host(k).view(np.uint8), want_k.view(np.uint8))
    assert np.array_equal(W.host(v).view(np.uint8), want_v.view(np.uint8))


@pytest.mark.parametrize("n", [1, 64, 500])
def test_swap_out_and_in_through_pinned_host_memory(cuda_dev, n):
    gen = torch.Generator().manual_seed(7 + n)
    nb, nh, bs, Hkv, D = n + 50, n + 30, 16, 8, 128
    k = _pool(nb, bs, Hkv, D, torch.bfloat16, cuda_dev, gen)
    v = _pool(nb, bs, Hkv, D, torch.bfloat16, cuda_dev, gen)
    hk = torch.zeros((nh, bs, Hkv, D), dtype=torch.bfloat16).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    rng = np.random.default_rng(n)
    out = np.stack([rng.permutation(nb)[:n], rng.permutation(nh)[:n]], 1).astype(np.int64)
    want_hk, want_hv = W.host(hk).copy(), W.host(hv).copy()
    M.copy_blocks(W.host(k), W.host(v), want_hk, want_hv, out)
    pkv.paged_kv_swap_blocks(k, v, hk, hv, torch.from_numpy(out).to(cuda_dev))
    torch.cuda.synchronize()
    assert np.array_equal(W.host(hk).view(np.uint16), want_hk.view(np.uint16))
    assert np.array_equal(W.host(hv).view(np.uint16), want_hv.view(np.uint16))
    # ... and back into other device blocks.
    back = np.stack([out[:, 1], rng.permutation(nb)[:n]], 1).astype(np.int64)
    want_k, want_v = W.host(k).copy(), W.host(v).copy()
    M.copy_blocks(W.host(hk), W.host(hv), want_k, want_v, back)
    pkv.paged_kv_swap_blocks(hk, hv, k, v, torch.from_numpy(back).to(cuda_dev))
    torch.cuda.synchronize()
    assert np.array_equal(W.host(k).view(np.uint16), want_k.view(np.uint16))
    assert np.array_equal(W.host(v).view(np.uint16), want_v.view(np.uint16))


def test_swap_rejects_pageable_host_memory(cuda_dev):
    k = torch.zeros((4, 16, 1, 64), dtype=torch.float16, device=cuda_dev)
    hk = torch.zeros((4, 16, 1, 64), dtype=torch.float16)           # not pinned
    pairs = torch.tensor([[0, 1]], dtype=torch.int64, device=cuda_dev)
    with pytest.raises(pkv.PagedKVError) as e:
        pkv.paged_kv_swap_blocks(k, k, hk, hk, pairs)
    assert e.value.status == -10


class GpuPools:
    """Device pool (bf16 rows [Hkv, D]) written by paged_kv_append, copied by
    paged_kv_copy_blocks, swapped to a pinned host pool by paged_kv_swap_blocks."""

    def __init__(self, num_blocks, num_host_blocks, bs, row_shape, dev):
        self.dev = dev
        self.k = torch.full((num_blocks, bs) + row_shape, float("nan"), dtype=torch.bfloat16,
                            device=dev)
        self.v = torch.full_like(self.k, float("nan"))
        self.hk = torch.zeros((num_host_blocks, bs) + row_shape, dtype=torch.bfloat16).pin_memory()
        self.hv = torch.zeros_like(self.hk).pin_memory()

    def write(self, slots, k_rows, v_rows):
        if len(slots) == 0:
            return
        key = torch.from_numpy(np.stack(k_rows)).to(torch.bfloat16).to(self.dev)
        val = torch.from_numpy(np.stack(v_rows)).to(torch.bfloat16).to(self.dev)
        sl = torch.as_tensor(np.asarray(slots, dtype=np.int64)).to(self.dev)
        pkv.paged_kv_append(key, val, self.k, self.v, sl)

    def _map(self, pairs):
        return torch.from_numpy(np.ascontiguousarray(pairs, dtype=np.int64)).to(self.dev)

    def copy(self, pairs):
        pkv.paged_kv_copy_blocks(self.k, self.v, self._map(pairs))

    def swap_out(self, pairs):
        if len(pairs):
            pkv.paged_kv_swap_blocks(self.k, self.v, self.hk, self.hv, self._map(pairs))
            torch.cuda.synchronize()

    def swap_in(self, pairs):
        if len(pairs):
            pkv.paged_kv_swap_blocks(self.hk, self.hv, self.k, self.v, self._map(pairs))

    def device_pools(self):
        torch.cuda.synchronize()
        return self.k.float().cpu().numpy(), self.v.float().cpu().numpy()


def _bf16(a):
    return torch.from_numpy(a).to(torch.bfloat16).float().numpy()


@pytest.mark.parametrize("prefix", [False, True])
@pytest.mark.parametrize("seed", [0, 1])
def test_managed_trace_on_the_gpu(cuda_dev, prefix, seed):
    bs, Hkv, D, Hq = 16, 2, 64, 8
    pools = GpuPools(160, 80, bs, (Hkv, D), cuda_dev)
    tr = Trace(pools, num_blocks=160, bs=bs, num_host_blocks=80, prefix_caching=prefix,
               row_shape=(Hkv, D), seed=seed, quantize=_bf16)
    for i in range(400):
        tr.step()
        if i % 50 == 49:
            tr.check_ledger()
            tr.check_contents(*pools.device_pools())
    st = tr.stats
    assert st["cow"] > 0 and st["swap_out"] > 0
    # Decode every resident sequence through the manager's block tables, and
    # compare with the oracle over the same rows laid out without paging.
    ids, table, lens = tr.tables()
    ids = [s for s, L in zip(ids, lens) if L > 0]
    ids, table, lens = tr.tables(ids)
    S = len(ids)
    q = torch.randn((S, Hq, D), generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
    out = torch.empty((S, Hq, D), dtype=torch.bfloat16, device=cuda_dev)
    P = 32
    msl = int(lens.max())
    ws = torch.empty(max(pkv.paged_attention_workspace_size(S, Hq, Hkv, D, msl, P), 1),
                     dtype=torch.uint8, device=cuda_dev)
    pkv.paged_attention_decode(out, q.to(cuda_dev), pools.k, pools.v,
                               torch.from_numpy(table).to(cuda_dev),
                               torch.from_numpy(lens).to(cuda_dev), max_seq_len=msl,
                               scale=D ** -0.5, partition_size=P, workspace=ws)
    torch.cuda.synchronize()
    # Unpaged layout of the model's rows: sequence i in its own run of blocks.
    nbs = [M.blocks_needed(int(L), bs) for L in lens]
    flat_k = np.zeros((sum(nbs), bs, Hkv, D), np.float32)
    flat_v = np.zeros_like(flat_k)
    ftable = np.full((S, max(nbs)), -1, np.int32)
    base = 0
    for i, s in enumerate(ids):
        k, v = tr.model.rows(s)
        L = len(k)
        for t in range(L):
            flat_k[base + t // bs, t % bs] = k[t]
            flat_v[base + t // bs, t % bs] = v[t]
        ftable[i, :nbs[i]] = np.arange(base, base + nbs[i])
        base += nbs[i]
    want, _ = oracle.decode(q.float().numpy(), flat_k, flat_v, ftable, lens.astype(np.int32),
                            num_heads=Hq, num_kv_heads=Hkv, head_dim=D, block_size=bs,
                            scale=D ** -0.5, q_dtype="f32", cache_dtype="f32")
    err = np.abs(out.float().cpu().numpy().astype(np.float64) - want)
    assert err.max() <= TOL["bf16"][0] and err.mean() <= TOL["bf16"][1], (err.max(), err.mean())


def test_shared_prefix_workload_from_the_manager(cuda_dev):
    # The FP8 shared-prefix shape with its sharing made by the block manager's
    # prefix cache: one 1024-token system prompt, private suffixes.
    bs, Hkv, Hq, D, S = 16, 8, 32, 128, 16
    rng = np.random.default_rng(5)
    system = list(rng.integers(0, 1000, size=1024))
    bm = BlockManager(S * 40 + 64, bs, prefix_caching=True)
    ids, cached = list(range(S)), []
    for s in ids:
        toks = system + list(rng.integers(0, 1000, size=int(rng.integers(16, 512))))
        _, c = bm.allocate(s, toks)
        cached.append(c)
    assert cached[0] == 0 and all(c == 1024 for c in cached[1:])
    table, lens = bm.block_tables(ids, 2048 // bs)
    assert (table[:, :1024 // bs] == table[0, :1024 // bs]).all()
    gen = torch.Generator().manual_seed(11)
    nb = bm.num_blocks
    kc = torch.randn((nb, bs, Hkv, D), generator=gen).to(torch.bfloat16).to(cuda_dev)
    vc = torch.randn((nb, bs, Hkv, D), generator=gen).to(torch.bfloat16).to(cuda_dev)
    q = torch.randn((S, Hq, D), generator=gen).to(torch.bfloat16).to(cuda_dev)
    out = torch.empty_like(q)
    msl = int(lens.max())
    ws = torch.empty(pkv.paged_attention_workspace_size(S, Hq, Hkv, D, msl, 256),
                     dtype=torch.uint8, device=cuda_dev)
    pkv.paged_attention_decode(out, q, kc, vc, torch.from_numpy(table).to(cuda_dev),
                               torch.from_numpy(lens).to(cuda_dev), max_seq_len=msl,
                               scale=D ** -0.5, partition_size=256, workspace=ws)
    torch.cuda.synchronize()
    want, _ = oracle.decode(W.host(q), W.host(kc), W.host(vc), table, lens, num_heads=Hq,
                            num_kv_heads=Hkv, head_dim=D, block_size=bs, scale=D ** -0.5,
                            q_dtype="bf16", cache_dtype="bf16")
    err = np.abs(out.float().cpu().numpy().astype(np.float64) - want)
    assert err.max() <= TOL["bf16"][0] and err.mean() <= TOL["bf16"][1]
